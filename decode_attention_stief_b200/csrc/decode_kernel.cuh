// decode_kernel.cuh -- split-KV decode attention over the latent (Stiefel-projected)
// KV cache, for sm_100a.
//
// Operation (StiefAttention technical summary, "Mecanismo Central" item 5): keys
// and values are stored as K_down = K P_K, V_down = V P_V and attention runs over
// the reconstructions K~ = K_down P_K^T, V~ = V_down P_V^T.  The kernel never forms
// K~ or V~; it uses the equal products
//     s_t = (q P_K) . K_down[t] / sqrt(d)          (query projected once per CTA)
//     o   = (sum_t softmax(s)_t V_down[t]) P_V^T   (up-projection after the mix)
// so the HBM stream is the bf16 latent cache, read once per KV head.
//
// One kernel, grid (splits, Hkv * qsub, B).  A CTA serves up to G_T <= 8 query heads
// of one KV head (a "unit") over one token range, with nwarps warps that each stream
// their own 32-token tiles (warp w takes tiles w, w + nwarps, ...) through a private
// ring of shared-memory stages.  Every stage holds the keys and the values of one tile,
// fetched by 2-D TMA tensor copies in 64/32/16-column pieces with the matching swizzle
// and completing on the stage's mbarrier.
//
// The contractions run on the warp-level tensor-core MMA (m16n8k16, bf16 operands,
// fp32 accumulators), with the query heads as the N = 8 dimension: column n of the
// MMA is head n & 3 for groups of up to 4 heads (part n >> 2), or head n with the part
// given by the n-tile for groups of 8.  Part 0 carries the bf16 rounding hi(x) of an
// fp32 operand x and part 1 its residual lo(x) = bf16(x - hi(x)); the two products are
// added in fp32, which keeps q~, the softmax weights and o~ at about 16 significant
// bits although the MMA takes bf16.  Per tile and warp:
//   scores  S[token][n]  = K_down[token][:] . Q^T[:][n]     (M = tokens, K = r_K)
//   online softmax over the tile (log2 domain, lazy rescale: accumulators are only
//   rescaled when a head's maximum passes its running reference by more than 8)
//   mix     O^T[dim][n] += V_down^T[dim][token] . P^T[token][n]  (M = r_V dims, K = tokens)
// where P^T comes from the score accumulators through an in-register 8x8 transpose
// (movmatrix).  The epilogue merges the warps (log-sum-exp); with one split it
// up-projects with P_V^T on the same MMA (M = d, K = r_V) and writes the output,
// otherwise it stores the latent partial state (o~, m, l) and takes a ticket: the last
// CTA of the unit merges the splits, up-projects once and resets the ticket counter,
// so the workspace counters stay zero between calls.
//
// Modes (compile-time, one instantiation each): the contiguous bf16 cache; the latent
// decode (q~ given, o~ returned: no base loads, projections or up-projection, for bases
// folded into the attention weights); paged caches (tiles addressed through a block
// table); int8 caches (the codes go straight into the integer MMA, m16n8k32 with s32
// accumulators: q~ and the softmax weights enter as 16-bit fixed point split into two 8-bit
// parts, per head and per head and tile respectively, so both products are exact in integers;
// the row scales multiply the scores and the weights).  Grids of more than one wave run two
// CTAs per SM with a smaller ring.
#pragma once

#include <cfloat>
#include <cmath>
#include <cstdint>

#include "stief_device.cuh"
#include "stief_internal.h"

namespace stief {

constexpr int kPreIssue = 1;         // stages per warp requested before the length is known
constexpr float kRescaleTau = 8.0f;  // lazy-rescale threshold (log2 units)
constexpr uint32_t kFull = 0xffffffffu;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// A bounded mbarrier wait whose outcome is the same in every lane of the warp (the
// warp-wide MMA and ldmatrix instructions that follow need all 32 lanes).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t* dev_status) {
  return __all_sync(kFull, mbar_wait_bounded(bar, parity, dev_status));
}

// ---------------------------------------------------------------------------- warp MMA

// Four 8x8 b16 matrices; lanes 8i..8i+7 give the row addresses of matrix i.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// Same, each matrix transposed on the way.
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// Transpose of an 8x8 b16 matrix held in the warp's registers (one pair per lane).
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// c += A(16x16, row) . B(16x8, col), bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// c = A . B (accumulators start at zero).
__device__ __forceinline__ void mma_bf16_z(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                           uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};"
      : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

// Two 8x8 b16 matrices (lanes 0-15 give the row addresses).
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}

// Integer products for the int8 caches, exact in s32:
// c (+)= A(16x32, s8, row) . B(32x8, s8 or u8, col)  and  c (+)= A(16x16, s8) . B(16x8, s8).
// Register i of A holds 4 consecutive k of row (lane >> 2) + 8 (i & 1), k from
// 4 (lane & 3) + 16 (i >> 1); register i of B 4 consecutive k from 4 (lane & 3) + 16 i of
// column lane >> 2.
template <bool ZERO, bool BU8>
__device__ __forceinline__ void mma_i8_k32(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (ZERO && BU8)
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
  else if constexpr (ZERO)
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
  else if constexpr (BU8)
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
template <bool ZERO>
__device__ __forceinline__ void mma_i8_k16(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  if constexpr (ZERO)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
        "{%7,%7,%7,%7};"
        : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
        : "r"(a0), "r"(a1), "r"(b0), "r"(0));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
        "{%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(b0));
}
// 4-bit codes, two per byte (low nibble first): each byte's low / high nibble moved to the top
// of the byte, i.e. 16 x the signed code, as four s8 lanes.
__device__ __forceinline__ uint32_t nib_lo(uint32_t p) { return (p << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t nib_hi(uint32_t p) { return p & 0xF0F0F0F0u; }

// Exact conversions of small integers through the fp32 bit pattern (integer and fp32 adds instead
// of the conversion pipe): 12582912 = 1.5 * 2^23 is the fp32 whose integers [2^23, 2^24) have
// spacing 1, so for |x| < 2^22 the pattern 0x4B400000 + x is the fp32 value 12582912 + x.
__device__ __forceinline__ float i2f_small(int x) { return __int_as_float(x + 0x4B400000) - 12582912.f; }
// rint(w * f) for 0 <= w * f < 2^22: the sum with 12582912 rounds once to an integer (RNE).
__device__ __forceinline__ uint32_t rint_small(float w, float f) {
  return __float_as_uint(fmaf(w, f, 12582912.f)) - 0x4B400000u;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// hi / lo bf16 parts of an fp32 pair, packed (first element in the low half)
__device__ __forceinline__ uint32_t hi_pair(float x0, float x1) { return pack_bf16x2_rn(x0, x1); }
__device__ __forceinline__ uint32_t lo_pair(float x0, float x1, uint32_t hi) {
  return pack_bf16x2_rn(x0 - bf16lo(hi), x1 - bf16hi(hi));
}

// ---------------------------------------------------------------------------- tile addressing

// Where 16-byte column chunk `chunk` of a row lives inside a tile of `rows` rows stacked
// from the pieces of a matrix r 16-bit columns wide: r / 64 pieces 64 columns wide, then one
// 32 wide if r % 64 >= 32, then one 16 wide if r % 32 == 16 (the order the host plans them
// in).
struct PieceLoc {
  uint32_t off;  // piece offset in the tile
  uint32_t w;    // piece width (columns)
  uint32_t lc;   // chunk index inside the piece
};
__device__ __forceinline__ PieceLoc locate(int r, int rows, int chunk) {
  const int col = chunk * 8;
  const int x64 = r & ~63;
  const int x32 = x64 + (r - x64 >= 32 ? 32 : 0);
  PieceLoc pl;
  if (col < x64) {
    pl.w = 64u;
    pl.off = (uint32_t)((col >> 6) * rows * 128);
    pl.lc = (uint32_t)((col & 63) >> 3);
  } else if (col < x32) {
    pl.w = 32u;
    pl.off = (uint32_t)(x64 * rows * 2);
    pl.lc = (uint32_t)((col - x64) >> 3);
  } else {
    pl.w = 16u;
    pl.off = (uint32_t)(x32 * rows * 2);
    pl.lc = (uint32_t)((col - x32) >> 3);
  }
  return pl;
}
// The same for int8 rows, whose r_bytes are addressed as r = r_bytes / 2 16-bit columns (r a
// multiple of 8): after the pieces above, one 8 columns (16 bytes) wide if r % 16 == 8.
__device__ __forceinline__ PieceLoc locate_i8(int r, int rows, int chunk) {
  const int x16 = r & ~15;
  if (chunk * 8 < x16) return locate(x16, rows, chunk);
  PieceLoc pl;
  pl.w = 8u;
  pl.off = (uint32_t)(x16 * rows * 2);
  pl.lc = 0u;
  return pl;
}
// Byte offset of (row, chunk) under the piece's TMA swizzle: 128-byte rows XOR the chunk
// with row & 7, 64-byte rows with (row >> 1) & 3, 32-byte rows with (row >> 2) & 1; 16-byte
// rows are not swizzled (8 consecutive rows already fill the 32 banks).
__device__ __forceinline__ uint32_t swz(const PieceLoc& pl, int row) {
  const uint32_t sw = pl.w == 64u   ? (uint32_t)(row & 7)
                      : pl.w == 32u ? (uint32_t)((row >> 1) & 3)
                      : pl.w == 16u ? (uint32_t)((row >> 2) & 1)
                                    : 0u;
  return pl.off + (uint32_t)row * pl.w * 2u + ((pl.lc ^ sw) << 4);
}
// Lane row / chunk for an x4 ldmatrix of a 16x16 block read as an A operand:
//  - row-major (no transpose; the block's rows are the MMA's M): matrices
//    (rows 0-7, chunk 0), (rows 8-15, chunk 0), (rows 0-7, chunk 1), (rows 8-15, chunk 1)
//  - transposed (the block's rows are the MMA's K): matrices
//    (rows 0-7, chunk 0), (rows 0-7, chunk 1), (rows 8-15, chunk 0), (rows 8-15, chunk 1)
__device__ __forceinline__ int a_row(int lane) { return (lane & 7) + ((lane >> 3) & 1) * 8; }
__device__ __forceinline__ int a_chunk(int lane) { return lane >> 4; }
__device__ __forceinline__ int at_row(int lane) { return (lane & 7) + (lane >> 4) * 8; }
__device__ __forceinline__ int at_chunk(int lane) { return (lane >> 3) & 1; }

// B fragments (k-step ks) of X^T for an fp32 matrix X[head][col] in shared memory (row
// stride xs floats): column n = lane >> 2 of n-tile j is (head, part) as described at the
// top; k = cols 16 ks + 2 (lane & 3) + {0, 1} (first register) and + 8 (second).
// (split into the loads and the conversion, so that callers can put the loads of several
// k-steps in flight before the first conversion waits for them)
__device__ __forceinline__ uint32_t bfrag_addr(const float* X, int xs, int ks, int lane, int nb) {
  const int n = lane >> 2;
  const int head = nb == 1 ? (n & 3) : n;
  return smem_u32(X + head * xs + 16 * ks + 2 * (lane & 3));
}
template <int NB>
__device__ __forceinline__ void bfrag_from(float2 x, float2 y, int lane, uint32_t (&bf)[NB][2]) {
  const int n = lane >> 2;
  const uint32_t hx = hi_pair(x.x, x.y), hy = hi_pair(y.x, y.y);
  const uint32_t lx = lo_pair(x.x, x.y, hx), ly = lo_pair(y.x, y.y, hy);
  if constexpr (NB == 1) {
    const bool lo = (n >> 2) != 0;
    bf[0][0] = lo ? lx : hx;
    bf[0][1] = lo ? ly : hy;
  } else {
    bf[0][0] = hx;
    bf[0][1] = hy;
    bf[NB - 1][0] = lx;
    bf[NB - 1][1] = ly;
  }
}
template <int NB>
__device__ __forceinline__ void bfrag_hilo(const float* X, int xs, int ks, int lane,
                                           uint32_t (&bf)[NB][2]) {
  const uint32_t xa = bfrag_addr(X, xs, ks, lane, NB);
  bfrag_from<NB>(lds_f32x2(xa), lds_f32x2(xa + 32u), lane, bf);
}

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// Shared-memory carve-up (byte offsets from the dynamic base).
struct DecodeSmem {
  uint32_t bars;    // nwarps*nstage "full" and nwarps*nstage "empty" stage barriers, then
                    // the setup barrier (q and P_K, then P_V) and the new-row barrier
  uint32_t ml;      // [nwarps][8] (m, l); then [8] M, [8] L; then a flag
  uint32_t qraw;    // [G_T][d] bf16 query rows
  uint32_t newraw;  // append: the new token's k and v rows, bf16 [2][d]
  uint32_t newlat;  // append: its projected key and value rows, bf16 [rK] then [rV]
  uint32_t qt;      // [8][xs] fp32: q~ (prologue), o~ (epilogue)
  uint32_t pmat;    // P_K (prologue), then P_V: d rows, pieces, swizzled
  uint32_t region;  // per warp a ring of stages (keys then values of a tile); later the
                    // cross-warp reduction and the split-merge staging
  uint32_t region_bytes;
  uint32_t stage;  // bytes of one ring stage (a multiple of 1 KiB)
  // int8 caches: a stage holds the key codes [tile][rK] and, from q8_v, the value codes
  // [tile][rV], in column pieces like the bf16 tiles (the rows' bytes read as 16-bit
  // columns); the row scales are not staged (the consumer lanes load them)
  uint32_t q8_v;
  uint32_t total;
  int xs;  // row stride of qt in floats
};

// `code`: the cache form, 0 bf16 rows, 1 int8 codes (r bytes per row), 2 4-bit codes (r / 2).
__host__ __device__ inline DecodeSmem decode_smem_layout(int NW, int ns, int rK, int rV, int tile,
                                                          int code = 0) {
  DecodeSmem s;
  const int rmax = rK > rV ? rK : rV;
  uint32_t off = 0;
  s.bars = off;
  off = align_up(off + 8u * (2 * NW * ns + 2), 16);
  s.ml = off;
  off = align_up(off + 4u * (NW * 16 + 16 + 4), 16);
  s.qraw = off;
  off = align_up(off + 2u * 8u * 128u, 16);  // up to 8 heads of d = 128
  s.newraw = off;
  off = align_up(off + 2u * 2u * 128u, 16);
  s.newlat = off;
  off = align_up(off + 2u * (uint32_t)(rK + rV), 16);
  s.xs = rmax + 4;
  s.qt = off;
  off = align_up(off + 4u * 8u * s.xs, 1024);
  s.pmat = off;
  off += 256u * rmax;  // d = 128 rows x r bf16
  s.region = off;
  if (code) {
    const uint32_t kb = code == 1 ? (uint32_t)rK : (uint32_t)rK / 2u;  // code bytes per row
    const uint32_t vb = code == 1 ? (uint32_t)rV : (uint32_t)rV / 2u;
    s.q8_v = align_up((uint32_t)tile * kb, 1024);  // the swizzle patterns need 1 KiB alignment
    s.stage = align_up(s.q8_v + (uint32_t)tile * vb, 1024);
  } else {
    s.q8_v = 0;
    s.stage = (uint32_t)tile * (rK + rV) * 2u;  // a multiple of 1 KiB
  }
  s.region_bytes = (uint32_t)NW * ns * s.stage;
  off += s.region_bytes;
  s.total = off;
  return s;
}

// One CTA = nwarps consumer warps + 1 producer warp.  Lane w of the producer requests the
// tiles (TMA) of consumer warp w and refills its stages as the warp releases them; the
// consumer warps only compute.  NB: B n-tiles (1: up to 4 heads, 2: up to 8);
// NKS >= rK/16; NMV >= rV/16.
constexpr int kMaxConsumerWarps = 8;

// Kernel modes: the contiguous bf16 cache, the latent decode, paged caches, int8 caches, and
// joint value latents (one value row per token shared by the KV heads; full or latent output);
// the int8 fused step (append + decode) is its own int8 mode.  Each is its own instantiation,
// so a mode's branches cost the others nothing.
constexpr int kModePlain = 0, kModeLatent = 1, kModePaged = 2, kModeQ8 = 3, kModeJointV = 4,
              kModeLatentJointV = 5, kModeQ4 = 6, kModePagedQ8 = 7, kModeQ8Append = 8;

template <int NB, int NKS, int NMV, int TT, int MODE>
__global__ void __launch_bounds__((kMaxConsumerWarps + 1) * 32, 1)
    stief_decode_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr bool LAT = MODE == kModeLatent || MODE == kModeLatentJointV;
  constexpr bool PG = MODE == kModePaged || MODE == kModePagedQ8;
  constexpr bool Q8 = MODE == kModeQ8 || MODE == kModePagedQ8 || MODE == kModeQ8Append;
  constexpr bool Q4 = MODE == kModeQ4;
  // the new token's rows enter the tile: every bf16 mode that may append, and the int8 fused
  // step (the other integer modes never append)
  constexpr bool INJECT = !(Q8 || Q4) || MODE == kModeQ8Append;
  constexpr bool QI = Q8 || Q4;  // integer codes with row scales
  constexpr bool JV = MODE == kModeJointV || MODE == kModeLatentJointV;
  constexpr int kTile = TT;
  constexpr int MT = TT / 16;              // 16-token m-tiles (scores) / k-steps (mix) per tile
  // score k-steps / value m-tiles whose fragments are loaded together (fewer where the
  // accumulators already take many registers)
  constexpr int KG = NB == 1 && TT == 32 ? 2 : 1;
  constexpr int VG = NB == 1 && TT == 32 ? 2 : 1;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int NW = a.nwarps, ns = a.nstage;
  const int NT = (NW + 1) * 32;  // all threads, the producer warp included
  const bool producer = warp == NW;
  const int s_idx = blockIdx.x;              // split
  const int kvh = blockIdx.y / a.qsub;       // KV head
  const int qs = blockIdx.y - kvh * a.qsub;  // query sub-group of that head
  const int b = blockIdx.z;
  const int d = a.d, rK = a.rK, rV = a.rV, S = a.S, G_T = a.G_T;
  const int nks = rK >> 4, nmv = rV >> 4;
  const int h0 = kvh * a.G + qs * G_T;          // first query head of this CTA
  const int gcount = min(G_T, a.G - qs * G_T);  // valid query heads here
  const size_t unit = ((size_t)b * a.Hkv + kvh) * a.qsub + qs;
  // PG: paged caches (the contiguous instantiations carry no page lookups)
  const CacheRows cr{PG ? a.block_table : nullptr, a.max_pages, a.page_size, a.num_pages, a.Hkv,
                     a.L_max};

  const DecodeSmem L = decode_smem_layout(NW, ns, rK, rV, TT, Q8 ? 1 : Q4 ? 2 : 0);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);  // [NW][ns]: tile landed
  uint64_t* empty = full + NW * ns;                             // [NW][ns]: tile consumed
  uint64_t* setup_bar = empty + NW * ns;  // phase 0: q and P_K, phase 1: P_V
  uint64_t* newrow_bar = setup_bar + 1;   // append: the new value row is in shared memory
  float* ml = reinterpret_cast<float*>(smem + L.ml);
  float* fin = ml + NW * 16;  // [8] M, [8] L
  int* flag = reinterpret_cast<int*>(fin + 16);
  float* qt = reinterpret_cast<float*>(smem + L.qt);
  const int xs = L.xs;
  uint8_t* pmat = smem + L.pmat;
  // a stage: the key tile, then the value tile at kt_bytes
  const uint32_t kt_bytes = QI ? L.q8_v : (uint32_t)kTile * rK * 2u;
  const uint32_t st_bytes = Q8   ? (uint32_t)kTile * (rK + rV)
                            : Q4 ? (uint32_t)kTile * (rK + rV) / 2u
                                 : kt_bytes + (uint32_t)kTile * rV * 2u;

  // the swizzle patterns assume 1 KiB-aligned tiles
  if (((smem_u32(smem + L.pmat) | smem_u32(smem + L.region)) & 1023u) != 0) {
    if (tid == 0) report(a.dev_status, STIEF_DEV_SMEM_ALIGN);
    return;
  }
#ifdef STIEF_TEST_HOOKS
  const uint32_t stall = a.test_stall_bytes;  // test build: a setup phase that never completes
#else
  constexpr uint32_t stall = 0u;
#endif
  if (tid == 0) {
    for (int i = 0; i < 2 * NW * ns + 2; ++i) mbar_init(&full[i], 1);
    flag[1] = 0;  // set when a wait for the setup phase (q, P_K, new rows) gave up
    fence_barrier_init();
    if (!LAT) {
      // P_K is requested before the dependency wait (its latency then overlaps the preceding
      // kernel's tail): a weight, which the calls document the preceding kernel must not
      // write.  Its bytes are added to the setup barrier's phase; q arrives after the wait.
      asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(setup_bar)),
                   "r"(2u * d * rK + stall) : "memory");
      const uint64_t keep = l2_policy_evict_last();
      for (int p = 0; p < a.ppk.n; ++p)
        tma_load_2d(pmat + a.ppk.p[p].smem_off, &a.maps[a.ppk.p[p].map], a.ppk.p[p].x, kvh * d,
                    setup_bar, keep);
    }
  }
  // the tensor maps are kernel parameters, not inputs: bring them in before the wait
  if (producer && lane < 12 && lane < a.nmaps) prefetch_tensormap(&a.maps[lane]);
  __syncthreads();

  // ---- split range and tiles --------------------------------------------------------------
  // Splits partition [0, S * chunk) by the host bound max_seq_len (the grid was sized by it),
  // so the first tiles can be requested before seq_lens has been read.  Consumer warp w takes
  // the split's tiles w, w + NW, ...
  const int t0 = s_idx * a.chunk;
  const int t_spec = min(t0 + a.chunk, a.max_seq_len);
  const int spec_tiles = t_spec > t0 ? (t_spec - t0 + kTile - 1) / kTile : 0;
  auto warp_tiles = [NW](int w, int tiles) { return w < tiles ? (tiles - w + NW - 1) / NW : 0; };
  // a tile's first row (tiles never straddle a page: page_size is a multiple of the tile);
  // a tile of an unmapped page is requested past the end of the pool, which the copy fills
  // with zeros (such tokens lie past the sequence and are masked)
  const long long pool_rows = PG ? (long long)a.num_pages * a.Hkv * a.page_size
                                 : (long long)a.B * a.Hkv * a.L_max;
  auto tile_row = [&](int t, bool before_wait = false) {
    const long long r = cache_row(cr, b, kvh, t, before_wait);
    return (int)(r < 0 ? pool_rows : r);
  };
  // TMA parameters of the cache pieces (at most three per matrix), kept in registers
  const void* kmap[3];
  const void* vmap[3];
  int kx[3], vx[3];
  uint32_t ko[3], vo[3];
#pragma unroll
  for (int p = 0; p < 3; ++p) {
    const int pk = p < a.pk.n ? p : 0, pv = p < a.pv.n ? p : 0;
    kmap[p] = &a.maps[a.pk.p[pk].map];
    kx[p] = a.pk.p[pk].x;
    ko[p] = (uint32_t)a.pk.p[pk].smem_off;
    vmap[p] = &a.maps[a.pv.p[pv].map];
    vx[p] = a.pv.p[pv].x;
    vo[p] = kt_bytes + (uint32_t)a.pv.p[pv].smem_off;
  }
  const int npk = a.pk.n, npv = a.pv.n;
  auto issue = [&](int w, int k, uint64_t policy, bool before_wait = false) {  // producer: tile k of consumer warp w
    uint8_t* dst = smem + L.region + ((size_t)w * ns + (k % ns)) * L.stage;
    uint64_t* bar = &full[w * ns + (k % ns)];
    // whole boxes land (rows past the sequence are masked on chip)
    mbar_arrive_expect_tx(bar, st_bytes);
    const int tt = t0 + (w + k * NW) * kTile;
    const int y = tile_row(tt, before_wait);
    // joint values: the value rows of sequence b are b * L_max + t, whatever the KV head
    const int yv = JV ? b * a.L_max + tt : y;
#pragma unroll
    for (int p = 0; p < 3; ++p)
      if (p < npk) tma_load_2d(dst + ko[p], kmap[p], kx[p], y, bar, policy);
#pragma unroll
    for (int p = 0; p < 3; ++p)
      if (p < npv) tma_load_2d(dst + vo[p], vmap[p], vx[p], yv, bar, policy);
  };

  // Every warp's first tile is requested before the dependency wait, like P_K, so that it
  // streams while the preceding kernel finishes (requesting whole rings there measured
  // slower: the flood delays q and some CTAs' data by microseconds).  The calls document that
  // the kernel immediately preceding them must not write the cache rows below the lengths
  // (nor, for page pools, the block-table entries of their pages), except, for bf16
  // per-head caches, the row just below each length (the one a preceding fused step on the
  // same caches appends), which is read again after the wait.  After an int8 fused step the
  // host clears `early` for the next decode in the stream, as after a compress.  Paged caches look the early
  // tiles' pages up around the L1 cache, so that no line read before the wait can hide an
  // entry the preceding kernel writes.  Right after a compress of this library (whose new
  // rows may still be in flight) the host clears `early` and nothing is requested before the
  // wait.
  const bool early_tiles = a.early != 0;
  int ring_issued = 0;  // producer lane w: tiles [0, ring_issued) of warp w are requested
  if (early_tiles && producer && lane < NW) {
    const uint64_t stream = l2_policy_evict_first();
    ring_issued = min(min(kPreIssue, ns), warp_tiles(lane, spec_tiles));
    for (int k = 0; k < ring_issued; ++k) issue(lane, k, stream, true);
  }
  // inputs may come from the preceding kernel in the stream: read nothing else before this
  pdl_wait();
  // the next kernel in the stream may be scheduled now (its CTAs take SMs as ours exit)
  pdl_launch_dependents();

  // q is requested before the length is read (its latency then overlaps the length's): the
  // producer's lane 0 sends q (its bytes join P_K's on the setup barrier, whose one arrival
  // waits for the length; the latent mode's q~ rows complete the barrier at once).  The other
  // modes' warps get their first tile now by the host bound and the rest of the rings once q
  // has landed (requested with it, their flood of misses would hold up q's copy).  Tiles past
  // the sequence are never consumed and are waited for before the ring is reused.
  if (producer) {
    if (lane == 0 && LAT) {
      mbar_arrive_expect_tx(setup_bar, 2u * gcount * rK + stall);
      bulk_g2s(smem + L.qraw, a.q + ((size_t)b * a.Hq + h0) * rK, 2u * gcount * rK, setup_bar);
    } else if (lane == 0) {
      asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(setup_bar)),
                   "r"(2u * gcount * d) : "memory");
      bulk_g2s(smem + L.qraw, a.q + ((size_t)b * a.Hq + h0) * d, 2u * gcount * d, setup_bar);
    }
    if (!early_tiles && lane < NW) {
      const uint64_t stream = l2_policy_evict_first();
      ring_issued = min(min(kPreIssue, ns), warp_tiles(lane, spec_tiles));
      for (int k = 0; k < ring_issued; ++k) issue(lane, k, stream);
    }
    __syncwarp();
  }

  int Lb = __ldcg(a.seq_lens + b);
  if (Lb < 0 || Lb > a.max_seq_len) {
    if (tid == 0 && s_idx == 0 && blockIdx.y == 0) report(a.dev_status, STIEF_DEV_BAD_LENGTH);
    Lb = 0;
  }
  // append path: the new token becomes row Lb and is attended to, when the cache has room
  // (Lb + 1 <= L_max; the host bound max_seq_len must cover the grown length too)
  bool appended = false;
  if (a.append) {
    if (Lb + 1 > a.L_max) {
      if (tid == 0 && s_idx == 0 && blockIdx.y == 0) report(a.dev_status, STIEF_DEV_CAPACITY_OVERFLOW);
    } else if (Lb + 1 > a.max_seq_len) {
      if (tid == 0 && s_idx == 0 && blockIdx.y == 0) report(a.dev_status, STIEF_DEV_BAD_LENGTH);
    } else if (PG && cache_row(cr, b, kvh, Lb) < 0) {  // the new token's page is not mapped
      if (tid == 0 && s_idx == 0 && blockIdx.y == 0) report(a.dev_status, STIEF_DEV_CAPACITY_OVERFLOW);
    } else {
      appended = true;
    }
  }
  const long long new_row = appended ? cache_row(cr, b, kvh, Lb) : 0;  // the appended row
  const int L_att = Lb + (appended ? 1 : 0);  // tokens attended to
  const bool owns_new = appended && Lb >= t0 && Lb < t0 + a.chunk;  // the new token is in range
  const int t1 = min(t0 + a.chunk, L_att);
  // append path: each CTA of a sequence takes a ticket once it has read the old length;
  // the CTA holding the last ticket (every CTA of the sequence has read it by then) stores
  // the grown length.  The ticket is requested here by an idle producer lane and only looked
  // at when the producer is done, so its round trip is off every critical path.
  const bool seq_lane = a.append && warp == NW && lane == 31;
  uint32_t seq_ticket = 0u;
  if (seq_lane) seq_ticket = atomicAdd(a.ws_seq + b, 1u);
  auto finish_sequence = [&]() {
    if (seq_lane && seq_ticket == (uint32_t)gridDim.x * gridDim.y - 1u) {
      a.ws_seq[b] = 0u;
      if (appended) a.seq_lens_w[b] = Lb + 1;
    }
  };
  const int n_tiles = t1 > t0 ? (t1 - t0 + kTile - 1) / kTile : 0;
  // int8 caches: the row scales of a tile come by coalesced loads, requested one tile ahead
  // (a TMA or bulk copy per tile costs more than its bytes): lane i holds the scales of
  // tokens i + 32 j of the tile.  The first tile's are requested before the setup wait.
  constexpr int SJ = QI ? TT / 32 : 1;
  float skc[SJ], svc[SJ], skn[SJ], svn[SJ];
  auto load_scales = [&](int kk) {
    if (kk < warp_tiles(warp, n_tiles)) {
      // (a consumed tile lies below the length: its page is mapped and holds the whole tile)
      const long long row = max(cache_row(cr, b, kvh, t0 + (warp + kk * NW) * kTile), 0ll) + lane;
#pragma unroll
      for (int j = 0; j < SJ; ++j) {
        skn[j] = __ldg(a.k_scale + row + 32 * j);
        svn[j] = __ldg(a.v_scale + row + 32 * j);
      }
    }
  };
  // ---- prologue ------------------------------------------------------------------------------
  bool ok = true;
  if (producer) {
    if (LAT) {
      // latent decode: the rows of q~ (requested above) are the input; no new rows, no append
    } else if (lane == 0) {
      // the new rows of the fused step follow once the length says which CTA holds the new
      // token: their bytes and the barrier's one arrival are added then
      if (owns_new) {
        mbar_arrive_expect_tx(setup_bar, 4u * d);
        const size_t row = ((size_t)b * a.Hkv + kvh) * d;
        bulk_g2s(smem + L.newraw, a.k_new + row, 2u * d, setup_bar);
        bulk_g2s(smem + L.newraw + 2u * d, a.v_new + row, 2u * d, setup_bar);
      } else {
        mbar_arrive(setup_bar);
      }
    }
    __syncwarp();
    if (lane < NW) {  // the rest of warp w's ring, as soon as q has landed
      const int want = min(ns, warp_tiles(lane, n_tiles));
      if (want > ring_issued && mbar_wait_bounded(setup_bar, 0u, nullptr)) {
        const uint64_t stream = l2_policy_evict_first();
        for (int k = ring_issued; k < want; ++k) issue(lane, k, stream);
        ring_issued = want;
      }
    }
    __syncwarp();
  } else if (LAT) {
    // q~ is given (bf16 [heads][r_K]): widen and scale it into log2 units; absent heads are 0
    ok = warp_wait(setup_bar, 0, a.dev_status);
    if (!ok && lane == 0) flag[1] = 1;
    const uint16_t* qr = reinterpret_cast<const uint16_t*>(smem + L.qraw);
    for (int i = tid; i < 8 * rK; i += NW * 32) {
      const int h = i / rK, j = i - h * rK;
      qt[h * xs + j] = h < gcount ? bf16_to_f32(qr[h * rK + j]) * a.qscale : 0.f;
    }
  } else {
    // q~ = q P_K on the MMA: q~^T[j][head] = sum_i P_K[i][j] q[head][i]
    // (M = the r_K columns of P_K, N = 8 heads, K = d), scaled into log2 units
    const int n = lane >> 2;  // B column = head
    if constexpr (QI) load_scales(0);
    ok = warp_wait(setup_bar, 0, a.dev_status);
    if (!ok && lane == 0) flag[1] = 1;
    uint32_t qb[8][2];  // d / 16 k-steps (explicit shared loads issued together)
    const uint32_t qrowb = smem_u32(smem + L.qraw) + 4u * (uint32_t)(min(n, gcount - 1) * (d / 2) + (lane & 3));
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qb[ks][0] = lds_u32(qrowb + 32u * ks);
      qb[ks][1] = lds_u32(qrowb + 32u * ks + 16u);
    }
    if (n >= gcount) {  // absent heads are zero columns
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) qb[ks][0] = qb[ks][1] = 0u;
    }
    // append: the new key row k_down = k_new P_K is the same contraction with B column 0 =
    // k_new (fp32 accumulation, one rounding to bf16).  Tasks 0..nks-1 are the q~ m-tiles,
    // nks..2 nks-1 the k_down m-tiles; the warps share them out.
    const uint32_t* krow = reinterpret_cast<const uint32_t*>(smem + L.newraw);
    const int ntasks = owns_new ? 2 * nks : nks;
    for (int task = warp; task < ntasks && ok; task += NW) {
      const bool key = task >= nks;
      const int mt = key ? task - nks : task;
      const PieceLoc pl = locate(rK, d, 2 * mt + at_chunk(lane));
      uint32_t af[8][4];  // all eight k-steps' fragments in flight together
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) ldsm_x4_t(smem_u32(pmat) + swz(pl, 16 * ks + at_row(lane)), af[ks]);
      float c[4], c2[4];  // even and odd k-steps: two MMA chains of four
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t b0 = qb[ks][0], b1 = qb[ks][1];
        if (key) {
          b0 = n == 0 ? krow[8 * ks + (lane & 3)] : 0u;
          b1 = n == 0 ? krow[8 * ks + 4 + (lane & 3)] : 0u;
        }
        if (ks == 0) mma_bf16_z(c, af[ks], b0, b1);
        else if (ks == 1) mma_bf16_z(c2, af[ks], b0, b1);
        else if (ks & 1) mma_bf16(c2, af[ks], b0, b1);
        else mma_bf16(c, af[ks], b0, b1);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) c[e] += c2[e];
      const int j = 16 * mt + (lane >> 2), hh = 2 * (lane & 3);
      if (!key) {
        const uint32_t qtb = smem_u32(qt);
        sts_f32(qtb + 4u * (uint32_t)(hh * xs + j), c[0] * a.qscale);
        sts_f32(qtb + 4u * (uint32_t)((hh + 1) * xs + j), c[1] * a.qscale);
        sts_f32(qtb + 4u * (uint32_t)(hh * xs + j + 8), c[2] * a.qscale);
        sts_f32(qtb + 4u * (uint32_t)((hh + 1) * xs + j + 8), c[3] * a.qscale);
      } else if ((lane & 3) == 0) {  // column 0: k_down[j], k_down[j + 8]
        uint16_t* kl = reinterpret_cast<uint16_t*>(smem + L.newlat);
        kl[j] = f32_to_bf16_rn(c[0]);
        kl[j + 8] = f32_to_bf16_rn(c[2]);
        if (!QI && qs == 0) {  // the cache row itself (every sub-group computes the same
          // values; int8 caches get the row's codes from the producer)
          uint16_t* dst = a.k_lat_w + new_row * rK;
          dst[j] = kl[j];
          dst[j + 8] = kl[j + 8];
        }
      }
    }
  }
  // q~ is in shared memory and every read of P_K is done.  The consumers meet on named
  // barrier 1 without waiting for the producer (which may still be requesting the rest of the
  // rings), and tell it on barrier 2 that P_V may now replace P_K.
  if (producer) {
    named_bar_sync(2, NT);
  } else {
    named_bar_arrive(2, NT);
    named_bar_sync(1, NW * 32);
  }
  // After a timed-out setup wait the setup barrier's phase never completes: nothing may arrive
  // on it again (P_V is not requested, the new value row not projected) and nothing waits for
  // its next phase.  The result is then undefined and the status word says so.
  const bool setup_ok = flag[1] == 0;

  // this lane's two heads (hA, hB = hA + 1) and, for NB == 1, its part of the MMA columns
  const int hA = NB == 1 ? 2 * (lane & 1) : 2 * (lane & 3);
  const bool lo_lane = NB == 1 && (lane & 2) != 0;
  float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
  float oacc[NMV][NB][4];
#pragma unroll
  for (int mt = 0; mt < NMV; ++mt)
#pragma unroll
    for (int j = 0; j < NB; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) oacc[mt][j][e] = 0.f;

  if (producer) {
    // ---- producer: P_V, the rest of every ring, then refills as stages are released ----
    if (lane == 0 && !LAT && setup_ok) {
      fence_proxy_async_smem();  // P_V replaces P_K, read through the generic proxy above
      const uint64_t keep = l2_policy_evict_last();
      mbar_arrive_expect_tx(setup_bar, 2u * d * rV);
      for (int p = 0; p < a.ppv.n; ++p)
        tma_load_2d(pmat + a.ppv.p[p].smem_off, &a.maps[a.ppv.p[p].map], a.ppv.p[p].x, kvh * d,
                    setup_bar, keep);
    }
    __syncwarp();
    {
      // Lane w serves consumer warp w: tile k goes into the stage the warp released after
      // tile k - ns.  The lanes stay converged: every pass tests all their stages at once
      // (non-blocking) and issues whatever is free, so one slow warp holds up no other.
      const int w = lane;
      const uint64_t stream = l2_policy_evict_first();
      const int tiles_w = lane < NW ? warp_tiles(w, n_tiles) : 0;
      for (int kk = ring_issued; kk < min(ns, tiles_w); ++kk) issue(w, kk, stream);
      ring_issued = max(ring_issued, min(ns, tiles_w));
      int k = ns;
      uint64_t last_progress = global_timer_ns();
      // append: once P_V has landed, the new value row v_down = v_new P_V is projected on
      // the MMA (B column 0) into shared memory (and the cache) for the tile that holds it
      // (one 16-row m-tile per call, so the refills in between are not held up)
      int vrow_next = owns_new && setup_ok ? 0 : nmv;  // next m-tile of the new value row
      // int8 caches (fused step): the new token's bf16 key and value rows (shared memory)
      // become one fp32 scale each (max |x| / 127, IEEE division) and RNE codes, as the
      // compress kernels store them; codes [rK] then [rV] and the two scales go to the
      // new-row area (its k and v inputs are consumed by now), and to the cache row
      auto quantize_new_rows = [&]() {
        const uint16_t* lat = reinterpret_cast<const uint16_t*>(smem + L.newlat);
        int8_t* codes = reinterpret_cast<int8_t*>(smem + L.newraw);
        float* nsc = reinterpret_cast<float*>(smem + L.newraw + 256);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const int r = part ? rV : rK, off = part ? rK : 0;
          float amax = 0.f;
          for (int j = lane; j < r; j += 32) amax = fmaxf(amax, fabsf(bf16_to_f32(lat[off + j])));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
          const float scale = __fdiv_rn(amax, 127.f);
          for (int j = lane; j < r; j += 32) codes[off + j] = (int8_t)quantize_code(bf16_to_f32(lat[off + j]), scale);
          if (lane == 0) nsc[part] = scale;
        }
        __syncwarp();
        if (qs == 0) {  // the cache rows (every sub-group computes the same values)
          int8_t* kq = reinterpret_cast<int8_t*>(a.k_lat_w) + new_row * rK;
          int8_t* vq = reinterpret_cast<int8_t*>(a.v_lat_w) + new_row * rV;
          for (int j = lane; j < rK; j += 32) kq[j] = codes[j];
          for (int j = lane; j < rV; j += 32) vq[j] = codes[rK + j];
          if (lane == 0) {
            a.k_scale_w[new_row] = nsc[0];
            a.v_scale_w[new_row] = nsc[1];
          }
        }
        __syncwarp();
      };
      auto project_vrow = [&]() {
        const uint32_t* vrow = reinterpret_cast<const uint32_t*>(smem + L.newraw + 2u * d);
        const bool vcol = (lane >> 2) == 0;  // lanes holding B column 0
        uint16_t* vl = reinterpret_cast<uint16_t*>(smem + L.newlat) + rK;
        {
          const int mv = vrow_next;
          float cv[4];
          const PieceLoc pl = locate(rV, d, 2 * mv + at_chunk(lane));
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            uint32_t af[4];
            ldsm_x4_t(smem_u32(pmat) + swz(pl, 16 * ks + at_row(lane)), af);
            const uint32_t v0 = vcol ? vrow[8 * ks + (lane & 3)] : 0u;
            const uint32_t v1 = vcol ? vrow[8 * ks + 4 + (lane & 3)] : 0u;
            if (ks == 0) mma_bf16_z(cv, af, v0, v1);
            else mma_bf16(cv, af, v0, v1);
          }
          if ((lane & 3) == 0) {  // column 0: v_down[j], v_down[j + 8]
            const int j = 16 * mv + (lane >> 2);
            vl[j] = f32_to_bf16_rn(cv[0]);
            vl[j + 8] = f32_to_bf16_rn(cv[2]);
            if (!QI && qs == 0) {
              a.v_lat_w[new_row * rV + j] = vl[j];
              a.v_lat_w[new_row * rV + j + 8] = vl[j + 8];
            }
          }
        }
        if (++vrow_next == nmv) {
          __syncwarp();
          if constexpr (MODE == kModeQ8Append) quantize_new_rows();
          if (lane == 0) mbar_arrive(newrow_bar);  // release: the row is visible to the consumers
        }
      };
      while (__any_sync(kFull, k < tiles_w)) {
        if (vrow_next < nmv && mbar_test(setup_bar, 1u)) project_vrow();
        const bool ready = k < tiles_w && mbar_test(&empty[w * ns + (k % ns)], (uint32_t)((k / ns - 1) & 1));
        if (ready) {
          issue(w, k, stream);
          ++k;
        }
        if (__any_sync(kFull, ready)) {
          last_progress = global_timer_ns();
        } else {
          __nanosleep(64);
          if (global_timer_ns() - last_progress > kWaitLimitNs) {  // the consumers gave up
            if (lane == 0) report(a.dev_status, STIEF_DEV_WAIT_TIMEOUT);
            break;
          }
        }
      }
      if (vrow_next < nmv && mbar_wait_bounded(setup_bar, 1u, a.dev_status))
        while (vrow_next < nmv) project_vrow();
      finish_sequence();
      // Every copy this lane requested must land before the region is reused or the CTA
      // exits: tiles requested before seq_lens was known but past the sequence are never
      // consumed, and after a timeout the consumers may have stopped early.  Only the last
      // tile requested into a stage can still be in flight (an earlier one was consumed
      // before the stage was refilled): wait for those (at once when they were consumed).
      if (lane < NW) {
        const int hi = k > ns ? k : ring_issued;  // tiles [0, hi) were requested
        for (int kk = max(0, hi - ns); kk < hi; ++kk)
          mbar_wait_bounded(&full[w * ns + kk % ns], (uint32_t)((kk / ns) & 1), nullptr);
      }
    }
    __syncwarp();
  } else {
    // ---- consumers: stream the warp's tiles ------------------------------------------------
    const int my_tiles = warp_tiles(warp, n_tiles);
    uint8_t* ring = smem + L.region + (size_t)warp * ns * L.stage;
    // int8 / 4-bit caches: a row's bytes are addressed as 16-bit columns (r / 2 or r / 4 of
    // them); the scores take k-steps of 32 codes (int8: the last one 16 when r_K % 32 == 16)
    const int rKc = Q8 ? rK / 2 : Q4 ? rK / 4 : rK, rVc = Q8 ? rV / 2 : Q4 ? rV / 4 : rV;
    const int nks8 = (rK + 31) >> 5;

    uint32_t qf[NKS][NB][2];       // bf16 caches: B fragments of Q^T (hi / lo parts)
    uint32_t qf8[NKS / 2][NB][2];  // int8 / 4-bit caches: the same as 8-bit parts
    float sqA = 0.f, sqB = 0.f;    // int8 / 4-bit caches: fixed-point scales of q~, heads hA, hA + 1
    if constexpr (!QI) {
      float2 qx[NKS], qy[NKS];
#pragma unroll
      for (int ks = 0; ks < NKS; ++ks)
        if (ks < nks) {
          const uint32_t xa = bfrag_addr(qt, xs, ks, lane, NB);
          qx[ks] = lds_f32x2(xa);
          qy[ks] = lds_f32x2(xa + 32u);
        }
#pragma unroll
      for (int ks = 0; ks < NKS; ++ks)
        if (ks < nks) bfrag_from<NB>(qx[ks], qy[ks], lane, qf[ks]);
    } else {
      // q~ in 16-bit fixed point per head, q16 = rint(q~ / s_q) with s_q = max_j |q~_j| / 32512,
      // split as q16 = 256 hi + lo (hi in [-127, 127], lo in [-128, 127]), so that a score is
      // s_q k_scale (256 K.hi + K.lo) with both integer products exact.  B column n carries
      // part n >> 2 of head n & 3 (groups of up to 4) or, for groups of 8, n-tile 0 the hi and
      // n-tile 1 the lo parts of head n.  4-bit caches: the key fragments carry 16 x the codes
      // (s_q takes the 1/16) and their k order within a k-step is the nibble order: register 0
      // slot i is column 8 (lane & 3) + 2 i, register 1 slot i column 8 (lane & 3) + 2 i + 1.
      const int n = lane >> 2;
      const int hcol = NB == 1 ? (n & 3) : n;
      const uint32_t qrow = smem_u32(qt) + 4u * (uint32_t)(hcol * xs);
      float amax = 0.f;
      for (int j = lane & 3; j < rK; j += 4) amax = fmaxf(amax, fabsf(lds_f32(qrow + 4u * (uint32_t)j)));
      amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
      const float inv = amax > 0.f ? 32512.f / amax : 0.f;  // absent heads are zero rows
      const float sq = amax * (1.f / 32512.f) * (Q4 ? 0.0625f : 1.f);
      sqA = __shfl_sync(kFull, sq, 4 * hA);  // lanes 4 h .. 4 h + 3 hold column h: head h
      sqB = __shfl_sync(kFull, sq, 4 * (hA + 1));
      const bool part_lo = NB == 1 && (n >> 2) != 0;
#pragma unroll
      for (int ks = 0; ks < NKS / 2; ++ks)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int k0 = Q4 ? 32 * ks + 8 * (lane & 3) : 32 * ks + 16 * half + 4 * (lane & 3);
          uint32_t hb = 0u, lb = 0u;
          if (ks < nks8 && k0 < rK) {
            float xv[4];
            if constexpr (Q4) {
              const float4 x0 = lds128f(qrow + 4u * (uint32_t)k0), x1 = lds128f(qrow + 4u * (uint32_t)(k0 + 4));
              xv[0] = half ? x0.y : x0.x;
              xv[1] = half ? x0.w : x0.z;
              xv[2] = half ? x1.y : x1.x;
              xv[3] = half ? x1.w : x1.z;
            } else {
              const float4 x = lds128f(qrow + 4u * (uint32_t)k0);
              xv[0] = x.x;
              xv[1] = x.y;
              xv[2] = x.z;
              xv[3] = x.w;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int q16 = __float2int_rn(xv[i] * inv);
              const int hi = (q16 + 128) >> 8, lo = q16 - hi * 256;
              hb |= ((uint32_t)hi & 0xffu) << (8 * i);
              lb |= ((uint32_t)lo & 0xffu) << (8 * i);
            }
          }
          if constexpr (NB == 1) {
            qf8[ks][0][half] = part_lo ? lb : hb;
          } else {
            qf8[ks][0][half] = hb;
            qf8[ks][NB - 1][half] = lb;
          }
        }
    }
    // ldmatrix lane offsets.  Keys: the x4 (x2 for a 16-wide k-step) of m-tile 0 of each
    // k-step, kstep bytes further per m-tile (4-bit: the x4 of rows 0-31 of the k-step's
    // 16-byte column, kstep further per 32 rows).  Values, bf16: the transposed x4 of each
    // 16-dim m-tile over tokens 0-15, vstep further per 16 tokens; int8: the transposed x4 of
    // rows (tokens) 0-31 of the m-tile's 16-byte column, vstep further per 32 tokens; 4-bit:
    // the same per 16-byte column (32 dims, two m-tiles).
    uint32_t koff[NKS], kstep[NKS], voff[NMV], vstep[NMV];
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks) {
      if (Q4) {
        const PieceLoc pl = locate_i8(rKc, kTile, min(ks, rKc / 8 - 1));
        koff[ks] = swz(pl, lane);
        kstep[ks] = 64u * pl.w;
        continue;
      }
      const int ch = min(2 * ks + a_chunk(lane), rKc / 8 - 1);
      const PieceLoc pl = QI ? locate_i8(rKc, kTile, ch) : locate(rKc, kTile, ch);
      koff[ks] = swz(pl, a_row(lane));
      kstep[ks] = 32u * pl.w;  // 16 rows further (the swizzle repeats every 8 rows)
    }
#pragma unroll
    for (int mt = 0; mt < NMV; ++mt) {
      if (QI) {
        const PieceLoc pl = locate_i8(rVc, kTile, min(mt, rVc / 8 - 1));
        voff[mt] = kt_bytes + swz(pl, lane);
        vstep[mt] = 64u * pl.w;
        continue;
      }
      const PieceLoc pl = locate(rV, kTile, 2 * mt + at_chunk(lane));
      voff[mt] = kt_bytes + swz(pl, at_row(lane));
      vstep[mt] = 32u * pl.w;
    }


    for (int k = 0; k < my_tiles && ok; ++k) {
      const int st = k % ns;
      if constexpr (QI) {
#pragma unroll
        for (int j = 0; j < SJ; ++j) {
          skc[j] = skn[j];
          svc[j] = svn[j];
        }
        load_scales(k + 1);
      }
      if (!warp_wait(&full[warp * ns + st], (uint32_t)((k / ns) & 1), a.dev_status)) {
        ok = false;
        break;
      }
      const uint32_t sbase = smem_u32(ring + (size_t)st * L.stage);
      const int tok0 = t0 + (warp + k * NW) * kTile;
      const int n = min(kTile, t1 - tok0);
      if (!QI && !JV && early_tiles && k < kPreIssue && Lb >= 1 && tok0 <= Lb - 1 && Lb - 1 < tok0 + kTile) {
        // this tile was requested before the dependency wait: the row just below the length
        // may have been appended by the preceding kernel (a fused step on the same caches),
        // so it is read again now (L2; the wait made it visible)
        const int r_prev = Lb - 1 - tok0;
        const long long prow = cache_row(cr, b, kvh, Lb - 1);
        for (int cch = lane; cch < (rK + rV) / 8; cch += 32) {
          const bool key = cch < rK / 8;
          const uint4 v = key ? __ldcg(reinterpret_cast<const uint4*>(a.k_lat_w + prow * rK) + cch)
                              : __ldcg(reinterpret_cast<const uint4*>(a.v_lat_w + prow * rV) + (cch - rK / 8));
          const PieceLoc pt = key ? locate(rK, kTile, cch) : locate(rV, kTile, cch - rK / 8);
          *reinterpret_cast<uint4*>(ring + (size_t)st * L.stage + (key ? 0u : kt_bytes) + swz(pt, r_prev)) = v;
        }
        fence_proxy_async_smem();  // generic writes into a stage the TMA engine fills
        __syncwarp();
      }
      if (INJECT && owns_new && tok0 <= Lb && Lb < tok0 + kTile) {
        // This tile holds the new token, whose cache rows were not written yet when the tile
        // was fetched: put the projected rows (key row from the prologue, value row from
        // the producer) into the tile.
        if (!warp_wait(newrow_bar, 0, a.dev_status)) {
          ok = false;
          break;
        }
        const int r_new = Lb - tok0;
        if constexpr (MODE == kModeQ8Append) {
          // the codes (16-byte chunks of the rows, addressed as 16-bit columns) and, in the
          // lane that holds the token's row scales, the scales
          const uint8_t* nc = smem + L.newraw;
          for (int cch = lane; cch < (rK + rV) / 16; cch += 32) {
            const bool key = cch < rK / 16;
            const PieceLoc pt = key ? locate_i8(rKc, kTile, cch) : locate_i8(rVc, kTile, cch - rK / 16);
            *reinterpret_cast<uint4*>(ring + (size_t)st * L.stage + (key ? 0u : kt_bytes) +
                                      swz(pt, r_new)) = *reinterpret_cast<const uint4*>(nc + 16 * cch);
          }
          const float* nsc = reinterpret_cast<const float*>(smem + L.newraw + 256);
#pragma unroll
          for (int j = 0; j < SJ; ++j)
            if (lane == (r_new & 31) && j == (r_new >> 5)) {
              skc[j] = nsc[0];
              svc[j] = nsc[1];
            }
        } else {
          const uint16_t* kl = reinterpret_cast<const uint16_t*>(smem + L.newlat);
          for (int cch = lane; cch < (rK + rV) / 8; cch += 32) {
            const bool key = cch < rK / 8;
            const PieceLoc pt = key ? locate(rK, kTile, cch) : locate(rV, kTile, cch - rK / 8);
            *reinterpret_cast<uint4*>(ring + (size_t)st * L.stage + (key ? 0u : kt_bytes) +
                                      swz(pt, r_new)) = *reinterpret_cast<const uint4*>(kl + 8 * cch);
          }
        }
        fence_proxy_async_smem();  // generic writes into a stage the TMA engine fills
        __syncwarp();
      }

      // Fragments are requested a group of k-steps (m-tiles) at a time, so their latencies
      // overlap; asm volatile keeps the order written here.
      // scores: s[mt][e] is token 16 mt + (lane >> 2) + 8 (e >> 1), head hA + (e & 1)
      float s[MT][4];
      uint32_t vf[VG][MT][4];  // bf16 caches: value fragments
      auto load_v = [&](int g0) {
#pragma unroll
        for (int u = 0; u < VG; ++u)
          if (g0 + u < nmv) {
#pragma unroll
            for (int kk = 0; kk < MT; ++kk)
              ldsm_x4_t(sbase + voff[g0 + u] + kk * vstep[g0 + u], vf[u][kk]);
          }
        if (n < kTile) {
          // the sequence ends inside this tile: the value rows past it may hold anything
          // (0 * NaN would reach the accumulators), so their fragment halves become zero.
          // Register r of a fragment holds tokens 16 kk + 8 (r >> 1) + 2 (lane & 3) + {0, 1}.
#pragma unroll
          for (int u = 0; u < VG; ++u)
#pragma unroll
            for (int kk = 0; kk < MT; ++kk)
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                const int tok = 16 * kk + 8 * (r >> 1) + 2 * (lane & 3);
                vf[u][kk][r] = tok + 1 < n ? vf[u][kk][r] : (tok < n ? (vf[u][kk][r] & 0xffffu) : 0u);
              }
        }
      };
      // int8 caches: value fragments of the first m-tiles (raw ldmatrix words, k32 steps)
      constexpr int VG8 = MT == 4 ? 1 : 2;
      uint32_t vx8[VG8][MT / 2][4];
      if constexpr (!QI) {
        // c[mt][j][e] is token 16 mt + (lane >> 2) + 8 (e >> 1), column 2 (lane & 3) + (e & 1)
        float c[MT][NB][4];
#pragma unroll
        for (int g0 = 0; g0 < NKS; g0 += KG)
          if (g0 < nks) {
            uint32_t kf[KG][MT][4];
#pragma unroll
            for (int u = 0; u < KG; ++u)
              if (g0 + u < nks) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
                  ldsm_x4(sbase + koff[g0 + u] + mt * kstep[g0 + u], kf[u][mt]);
              }
#pragma unroll
            for (int u = 0; u < KG; ++u)
              if (g0 + u < nks) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                  for (int j = 0; j < NB; ++j) {
                    if (g0 + u == 0) mma_bf16_z(c[mt][j], kf[u][mt], qf[0][j][0], qf[0][j][1]);
                    else mma_bf16(c[mt][j], kf[u][mt], qf[g0 + u][j][0], qf[g0 + u][j][1]);
                  }
              }
          }
        // value fragments do not depend on the scores: request the first group now
        load_v(0);
        // add the hi and lo parts
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            s[mt][e] = NB == 1 ? c[mt][0][e] + __shfl_xor_sync(kFull, c[mt][0][e], 2)
                               : c[mt][0][e] + c[mt][NB - 1][e];
      } else {
        // integer scores of the codes against the two parts of q~
        int ci[MT][NB][4];
#pragma unroll
        for (int ks = 0; ks < NKS / 2; ++ks)
          if (Q4 && ks < nks8) {
            // 4-bit: one x4 gives 32 rows of the k-step's 16-byte column; a byte's low and high
            // nibbles, moved to the top of the byte, are 16 x the two codes as exact s8
            uint32_t kp[MT / 2][4];
#pragma unroll
            for (int gq = 0; gq < MT / 2; ++gq) ldsm_x4(sbase + koff[ks] + gq * kstep[ks], kp[gq]);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              const uint32_t p0 = kp[mt >> 1][2 * (mt & 1)], p1 = kp[mt >> 1][2 * (mt & 1) + 1];
              const uint32_t af[4] = {nib_lo(p0), nib_lo(p1), nib_hi(p0), nib_hi(p1)};
#pragma unroll
              for (int j = 0; j < NB; ++j) {
                if (ks == 0) mma_i8_k32<true, false>(ci[mt][j], af, qf8[ks][j][0], qf8[ks][j][1]);
                else mma_i8_k32<false, false>(ci[mt][j], af, qf8[ks][j][0], qf8[ks][j][1]);
              }
            }
          } else if (!Q4 && ks < nks8) {
            const bool k32 = 32 * ks + 32 <= rK;
            uint32_t kf[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              if (k32) ldsm_x4(sbase + koff[ks] + mt * kstep[ks], kf[mt]);
              else ldsm_x2(sbase + koff[ks] + mt * kstep[ks], kf[mt][0], kf[mt][1]);
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
              for (int j = 0; j < NB; ++j) {
                if (k32) {
                  if (ks == 0) mma_i8_k32<true, false>(ci[mt][j], kf[mt], qf8[ks][j][0], qf8[ks][j][1]);
                  else mma_i8_k32<false, false>(ci[mt][j], kf[mt], qf8[ks][j][0], qf8[ks][j][1]);
                } else {
                  if (ks == 0) mma_i8_k16<true>(ci[mt][j], kf[mt][0], kf[mt][1], qf8[ks][j][0]);
                  else mma_i8_k16<false>(ci[mt][j], kf[mt][0], kf[mt][1], qf8[ks][j][0]);
                }
              }
          }
        // the first value m-tiles' (4-bit: 16-byte columns') fragments do not depend on the
        // scores: request them now
#pragma unroll
        for (int u = 0; u < VG8; ++u)
          if (Q4 ? 2 * u < nmv : u < nmv) {
#pragma unroll
            for (int kk = 0; kk < MT / 2; ++kk) ldsm_x4_t(sbase + voff[u] + kk * vstep[u], vx8[u][kk]);
          }
        // the tile's key scales: tokens 16 mt + (lane >> 2) + 8 h
        float skt[MT][2];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int h = 0; h < 2; ++h)
            skt[mt][h] = __shfl_sync(kFull, skc[(16 * mt + 8 * h) >> 5], ((16 * mt + 8 * h) & 31) + (lane >> 2));
        // s = s_q k_scale (256 hi + lo): each part is below 2^21 in magnitude (r <= 128 codes of
        // at most 127 times at most 128), so it converts exactly; the sum rounds once in fp32
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float v;
            const float fc = i2f_small(ci[mt][0][e]);
            if constexpr (NB == 1) {
              const float fo = __shfl_xor_sync(kFull, fc, 2);
              v = lo_lane ? fmaf(fo, 256.f, fc) : fmaf(fc, 256.f, fo);
            } else {
              v = fmaf(fc, 256.f, i2f_small(ci[mt][NB - 1][e]));
            }
            s[mt][e] = v * (skt[mt][e >> 1] * ((e & 1) ? sqB : sqA));
          }
      }
      if (n < kTile) {  // missing tokens take no weight
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (16 * mt + (lane >> 2) + 8 * (e >> 1) >= n) s[mt][e] = -INFINITY;
      }

      // online softmax, log2 domain.  The lane maxima are voted on first: only when some
      // head passes its reference by more than the threshold are the maxima over the 8
      // lanes sharing the heads formed and the accumulators rescaled.
      float tA = fmaxf(s[0][0], s[0][2]), tB = fmaxf(s[0][1], s[0][3]);
#pragma unroll
      for (int mt = 1; mt < MT; ++mt) {
        tA = fmaxf(tA, fmaxf(s[mt][0], s[mt][2]));
        tB = fmaxf(tB, fmaxf(s[mt][1], s[mt][3]));
      }
      if (__any_sync(kFull, tA > mA + kRescaleTau || tB > mB + kRescaleTau)) {
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          tA = fmaxf(tA, __shfl_xor_sync(kFull, tA, o));
          tB = fmaxf(tB, __shfl_xor_sync(kFull, tB, o));
        }
        if (tA > mA + kRescaleTau) {
          const float mn = fmaxf(mA, tA);
          const float f = ex2(mA - mn);  // 0 while mA is -inf
          lA *= f;
          mA = mn;
#pragma unroll
          for (int mt = 0; mt < NMV; ++mt)
#pragma unroll
            for (int j = 0; j < NB; ++j) {
              oacc[mt][j][0] *= f;
              oacc[mt][j][2] *= f;
            }
        }
        if (tB > mB + kRescaleTau) {
          const float mn = fmaxf(mB, tB);
          const float f = ex2(mB - mn);
          lB *= f;
          mB = mn;
#pragma unroll
          for (int mt = 0; mt < NMV; ++mt)
#pragma unroll
            for (int j = 0; j < NB; ++j) {
              oacc[mt][j][1] *= f;
              oacc[mt][j][3] *= f;
            }
        }
      }
      const float uA = mA == -INFINITY ? 0.f : mA, uB = mB == -INFINITY ? 0.f : mB;
      float pa_sum = 0.f, pb_sum = 0.f;
      if constexpr (!QI) {
        // weights of the tile as B fragments of P^T: block r = tokens 8r..8r+7 in the score
        // layout (row = token, columns = this lane's two heads), transposed to (token pairs, head)
        uint32_t pb[NB][2 * MT];
#pragma unroll
        for (int r = 0; r < 2 * MT; ++r) {
          const int mt = r >> 1, e0 = (r & 1) * 2;
          const float pA = ex2(s[mt][e0] - uA), pB = ex2(s[mt][e0 + 1] - uB);
          pa_sum += pA;
          pb_sum += pB;
          const uint32_t hw = hi_pair(pA, pB);
          const uint32_t lw = lo_pair(pA, pB, hw);
          if constexpr (NB == 1) {
            pb[0][r] = movm_t(lo_lane ? lw : hw);
          } else {
            pb[0][r] = movm_t(hw);
            pb[NB - 1][r] = movm_t(lw);
          }
        }
        lA += pa_sum;
        lB += pb_sum;
        // value mix: O^T[dim][n] += V^T[dim][token] P^T[token][n]
#pragma unroll
        for (int g0 = 0; g0 < NMV; g0 += VG)
          if (g0 < nmv) {
            if (g0 > 0) load_v(g0);
#pragma unroll
            for (int u = 0; u < VG; ++u)
              if (g0 + u < nmv) {
#pragma unroll
                for (int kk = 0; kk < MT; ++kk)
#pragma unroll
                  for (int j = 0; j < NB; ++j)
                    mma_bf16(oacc[g0 + u][j], vf[u][kk], pb[j][2 * kk], pb[j][2 * kk + 1]);
              }
          }
      } else {
        // int8 caches: a token's weight in the mix is p v_scale (the scale is not in l).  Per
        // head and tile the weights become 16-bit fixed point, w16 = rint(w / sigma) with
        // sigma = max w / 65535, split into two unsigned bytes (w16 = 256 hi + lo): the mix
        // of the codes against each part is exact in s32 and sigma (256 for the hi part)
        // brings it back into the fp32 accumulators.  Rows past the sequence take weight 0
        // whatever their scale holds.
        float svt[2 * MT];
#pragma unroll
        for (int r = 0; r < 2 * MT; ++r)
          svt[r] = __shfl_sync(kFull, svc[(16 * (r >> 1) + 8 * (r & 1)) >> 5],
                               ((16 * (r >> 1) + 8 * (r & 1)) & 31) + (lane >> 2));
        float wA[2 * MT], wB[2 * MT];
        float xA = 0.f, xB = 0.f;
#pragma unroll
        for (int r = 0; r < 2 * MT; ++r) {
          const int mt = r >> 1, e0 = (r & 1) * 2;
          const float pA = ex2(s[mt][e0] - uA), pB = ex2(s[mt][e0 + 1] - uB);
          pa_sum += pA;
          pb_sum += pB;
          const float sv = n < kTile && 16 * mt + (lane >> 2) + 8 * (r & 1) >= n ? 0.f : svt[r];
          wA[r] = pA * sv;
          wB[r] = pB * sv;
          xA = fmaxf(xA, wA[r]);
          xB = fmaxf(xB, wB[r]);
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          xA = fmaxf(xA, __shfl_xor_sync(kFull, xA, o));
          xB = fmaxf(xB, __shfl_xor_sync(kFull, xB, o));
        }
        lA += pa_sum;
        lB += pb_sum;
        const float fA = xA > 0.f ? 65535.f * rcp_approx(xA) : 0.f;
        const float fB = xB > 0.f ? 65535.f * rcp_approx(xB) : 0.f;
        // B fragments of W^T: per score m-tile, the lane's (token g, token g + 8) byte pairs of
        // its two columns, transposed (movmatrix) to 4 tokens of one column.  Register r of a
        // k32 step then holds tokens 2 (lane & 3) + {0, 8, 1, 9} + 16 r of column lane >> 2;
        // the value fragments below put their tokens in the same order.
        uint32_t pb8[NB][MT];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          // w16 = rint(w f) in [0, 65535] (w f <= 65535 (1 + 2^-22))
          const uint32_t a0 = rint_small(wA[2 * mt], fA), a1 = rint_small(wA[2 * mt + 1], fA);
          const uint32_t b0 = rint_small(wB[2 * mt], fB), b1 = rint_small(wB[2 * mt + 1], fB);
          const uint32_t u = __byte_perm(a0, b0, 0x5410), v = __byte_perm(a1, b1, 0x5410);
          // hi bytes: u.1 v.1 u.3 v.3; lo bytes: u.0 v.0 u.2 v.2
          if constexpr (NB == 1) {
            pb8[0][mt] = movm_t(__byte_perm(u, v, lo_lane ? 0x6240 : 0x7351));
          } else {
            pb8[0][mt] = movm_t(__byte_perm(u, v, 0x7351));
            pb8[NB - 1][mt] = movm_t(__byte_perm(u, v, 0x6240));
          }
        }
        // (4-bit: the value fragments carry 16 x the codes, so sigma takes 1/16)
        const float sA = xA * (Q4 ? 1.f / (16.f * 65535.f) : 1.f / 65535.f);
        const float sB = xB * (Q4 ? 1.f / (16.f * 65535.f) : 1.f / 65535.f);
        float zA[NB], zB[NB];  // sigma of the lane's two columns per n-tile (256 sigma: hi part)
#pragma unroll
        for (int j = 0; j < NB; ++j) {
          const bool hi = NB == 1 ? !lo_lane : j == 0;
          zA[j] = hi ? 256.f * sA : sA;
          zB[j] = hi ? 256.f * sB : sB;
        }
        if constexpr (Q4) {
        // 4-bit: the transposed x4 of a 16-byte column gives each lane, per 8 tokens, the bytes
        // 2 g (dims 4 g, 4 g + 1) and 2 g + 1 (dims 4 g + 2, 4 g + 3) of tokens 2 (lane & 3) + {0, 1};
        // byte permutes gather 4 tokens in the weights' order and the nibble masks split the
        // dims: m-tile 2 c has rows g = dim 4 g, g + 8 = dim 4 g + 1 of column c, m-tile 2 c + 1
        // rows g = dim 4 g + 2, g + 8 = dim 4 g + 3.
#pragma unroll
        for (int c0 = 0; c0 < NMV / 2; c0 += VG8)
          if (2 * c0 < nmv) {
            if (c0 > 0) {
#pragma unroll
              for (int u = 0; u < VG8; ++u)
                if (2 * (c0 + u) < nmv) {
#pragma unroll
                  for (int kk = 0; kk < MT / 2; ++kk)
                    ldsm_x4_t(sbase + voff[c0 + u] + kk * vstep[c0 + u], vx8[u][kk]);
                }
            }
#pragma unroll
            for (int u = 0; u < VG8; ++u)
              if (2 * (c0 + u) < nmv) {
                const int c = c0 + u;
                int accP[NB][4], accQ[NB][4];
#pragma unroll
                for (int kk = 0; kk < MT / 2; ++kk) {
                  const uint32_t* x = vx8[u][kk];
                  const uint32_t p0 = __byte_perm(x[0], x[1], 0x6240), q0 = __byte_perm(x[0], x[1], 0x7351);
                  const uint32_t p1 = __byte_perm(x[2], x[3], 0x6240), q1 = __byte_perm(x[2], x[3], 0x7351);
                  const uint32_t afP[4] = {nib_lo(p0), nib_hi(p0), nib_lo(p1), nib_hi(p1)};
                  const uint32_t afQ[4] = {nib_lo(q0), nib_hi(q0), nib_lo(q1), nib_hi(q1)};
#pragma unroll
                  for (int j = 0; j < NB; ++j) {
                    if (kk == 0) {
                      mma_i8_k32<true, true>(accP[j], afP, pb8[j][2 * kk], pb8[j][2 * kk + 1]);
                      mma_i8_k32<true, true>(accQ[j], afQ, pb8[j][2 * kk], pb8[j][2 * kk + 1]);
                    } else {
                      mma_i8_k32<false, true>(accP[j], afP, pb8[j][2 * kk], pb8[j][2 * kk + 1]);
                      mma_i8_k32<false, true>(accQ[j], afQ, pb8[j][2 * kk], pb8[j][2 * kk + 1]);
                    }
                  }
                }
#pragma unroll
                for (int j = 0; j < NB; ++j)
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const float z = (e & 1) ? zB[j] : zA[j];
                    oacc[2 * c][j][e] = fmaf(i2f_small(accP[j][e]), z, oacc[2 * c][j][e]);
                    oacc[2 * c + 1][j][e] = fmaf(i2f_small(accQ[j][e]), z, oacc[2 * c + 1][j][e]);
                  }
              }
          }
        } else {
        // value mix: the transposed x4 gives each lane, per 8 tokens, a 16-bit pair of dims
        // (2 g, 2 g + 1) of tokens 2 (lane & 3) + {0, 1}; byte permutes make A rows of 4 tokens
        // in the weights' order: row g is dim 2 g of the m-tile, row g + 8 dim 2 g + 1.
#pragma unroll
        for (int g0 = 0; g0 < NMV; g0 += VG8)
          if (g0 < nmv) {
            if (g0 > 0) {
#pragma unroll
              for (int u = 0; u < VG8; ++u)
                if (g0 + u < nmv) {
#pragma unroll
                  for (int kk = 0; kk < MT / 2; ++kk)
                    ldsm_x4_t(sbase + voff[g0 + u] + kk * vstep[g0 + u], vx8[u][kk]);
                }
            }
#pragma unroll
            for (int u = 0; u < VG8; ++u)
              if (g0 + u < nmv) {
                int acc[NB][4];
#pragma unroll
                for (int kk = 0; kk < MT / 2; ++kk) {
                  const uint32_t* x = vx8[u][kk];
                  const uint32_t af[4] = {__byte_perm(x[0], x[1], 0x6240), __byte_perm(x[0], x[1], 0x7351),
                                          __byte_perm(x[2], x[3], 0x6240), __byte_perm(x[2], x[3], 0x7351)};
#pragma unroll
                  for (int j = 0; j < NB; ++j) {
                    if (kk == 0) mma_i8_k32<true, true>(acc[j], af, pb8[j][2 * kk], pb8[j][2 * kk + 1]);
                    else mma_i8_k32<false, true>(acc[j], af, pb8[j][2 * kk], pb8[j][2 * kk + 1]);
                  }
                }
#pragma unroll
                for (int j = 0; j < NB; ++j)
#pragma unroll
                  for (int e = 0; e < 4; ++e)
                    // a tile's s32 mix is below 2^21 (64 tokens x 127 x 255): exact conversion
                    oacc[g0 + u][j][e] = fmaf(i2f_small(acc[j][e]), (e & 1) ? zB[j] : zA[j], oacc[g0 + u][j][e]);
              }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[warp * ns + st]);  // the stage may be refilled
    }
  }

  // ---- merge the warps ------------------------------------------------------------------
  // (a) every warp's running maximum and sum per head; (b) the CTA's maximum per head, to
  // which every warp rescales its accumulators; (c) sums over the warps (no exponentials).
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    lA += __shfl_xor_sync(kFull, lA, o);
    lB += __shfl_xor_sync(kFull, lB, o);
  }
  // o~ of (dim 16 mt + (lane >> 2) + 8 (e >> 1), head hA + (e & 1)); int8 caches: dim
  // 16 mt + 2 (lane >> 2) + (e >> 1); 4-bit caches: dim 32 (mt >> 1) + 4 (lane >> 2) +
  // 2 (mt & 1) + (e >> 1)
  float ov[NMV][4];
#pragma unroll
  for (int mt = 0; mt < NMV; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e)
      ov[mt][e] = NB == 1 ? oacc[mt][0][e] + __shfl_xor_sync(kFull, oacc[mt][0][e], 2)
                          : oacc[mt][0][e] + oacc[mt][NB - 1][e];
  const int HR = NB == 1 ? 4 : 8;  // heads the MMA columns carry
  if (!producer && !lo_lane && (lane >> 2) == 0) {
    ml[(warp * 8 + hA) * 2] = mA;
    ml[(warp * 8 + hA) * 2 + 1] = lA;
    ml[(warp * 8 + hA + 1) * 2] = mB;
    ml[(warp * 8 + hA + 1) * 2 + 1] = lB;
  }
  __syncthreads();  // every warp is done with its ring: the region becomes the reduction buffer
  float* red = reinterpret_cast<float*>(smem + L.region);  // [NW][8][rV]
  // (explicit shared accesses issued in batches: see lds_f32)
  const uint32_t mlb = smem_u32(ml), redb = smem_u32(red);
  if (!producer) {
    float va[kMaxConsumerWarps], vb[kMaxConsumerWarps];
#pragma unroll
    for (int w = 0; w < kMaxConsumerWarps; ++w) {
      const int ww = w < NW ? w : 0;  // a repeat of warp 0 changes no maximum
      va[w] = lds_f32(mlb + 8u * (uint32_t)(ww * 8 + hA));
      vb[w] = lds_f32(mlb + 8u * (uint32_t)(ww * 8 + hA + 1));
    }
    float MA = va[0], MB = vb[0];
#pragma unroll
    for (int w = 1; w < kMaxConsumerWarps; ++w) {
      MA = fmaxf(MA, va[w]);
      MB = fmaxf(MB, vb[w]);
    }
    const float fA = mA == -INFINITY ? 0.f : ex2(mA - MA);  // 0 for a warp that saw no token
    const float fB = mB == -INFINITY ? 0.f : ex2(mB - MB);
    if (!lo_lane) {
#pragma unroll
      for (int mt = 0; mt < NMV; ++mt)
        if (mt < nmv)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            sts_f32(redb + 4u * (uint32_t)((warp * 8 + hA + (e & 1)) * rV +
                                           (Q4   ? 32 * (mt >> 1) + 4 * (lane >> 2) + 2 * (mt & 1) + (e >> 1)
                                            : Q8 ? 16 * mt + 2 * (lane >> 2) + (e >> 1)
                                                 : 16 * mt + (lane >> 2) + 8 * (e >> 1))),
                    ov[mt][e] * ((e & 1) ? fB : fA));
      if ((lane >> 2) == 0) {  // the sums rescaled in place (only the maxima were read above)
        sts_f32(mlb + 8u * (uint32_t)(warp * 8 + hA) + 4u, lA * fA);
        sts_f32(mlb + 8u * (uint32_t)(warp * 8 + hA + 1) + 4u, lB * fB);
        if (warp == 0) {
          fin[hA] = MA;
          fin[hA + 1] = MB;
        }
      }
    }
  }
  __syncthreads();
  // o~ of the CTA (scaled to its maximum fin[h], normalised when this CTA finishes the unit
  // alone) and its sum: into qt and fin (the up-projection's operand, or the ticket merge's
  // partial state), or straight out as this split's tagged record
  const bool tagged_merge = S > 1 && a.merge_tagged;
  const int RW = rV + 2;  // words per tagged record: o~[rV], m, l
  uint64_t* my_words = tagged_merge ? a.ws_words + ((size_t)unit * S + s_idx) * G_T * RW : nullptr;
  for (int idx = tid; idx < HR * (rV / 2); idx += NT) {
    const int h = idx / (rV / 2), jj = 2 * (idx - h * (rV / 2));
    float2 v[kMaxConsumerWarps];
    float lw[kMaxConsumerWarps];
#pragma unroll
    for (int w = 0; w < kMaxConsumerWarps; ++w) {
      const int ww = w < NW ? w : 0;
      v[w] = lds_f32x2(redb + 4u * (uint32_t)((ww * 8 + h) * rV + jj));
      lw[w] = lds_f32(mlb + 8u * (uint32_t)(ww * 8 + h) + 4u);
    }
    float o0 = 0.f, o1 = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kMaxConsumerWarps; ++w)
      if (w < NW) {
        o0 += v[w].x;
        o1 += v[w].y;
        lsum += lw[w];
      }
    if (S == 1) {
      o0 = lsum > 0.f ? o0 / lsum : 0.f;
      o1 = lsum > 0.f ? o1 / lsum : 0.f;
    }
    if (tagged_merge) {
      if (h < gcount) {
        uint64_t* r = my_words + h * RW;
        st_tagged2(r + jj, tagged(o0, 1u), tagged(o1, 1u));
        if (jj == 0) st_tagged2(r + rV, tagged(fin[h], 1u), tagged(lsum, 1u));
      }
    } else {
      qt[h * xs + jj] = o0;
      qt[h * xs + jj + 1] = o1;
      if (jj == 0) fin[8 + h] = lsum;
    }
  }
  __syncthreads();

  // ---- up-projection o = o~ P_V^T on the MMA: o^T[i][n] = sum_j P_V[i][j] o~^T[j][n] ----
  // (M = d, N = heads, K = r_V) from the normalised o~ in qt; warp w takes rows 16 w,
  // 16 (w + NW + 1), ...
  auto up_project = [&](int nheads, int hbase, int hstride) {
    if (!setup_ok || !warp_wait(setup_bar, 1, a.dev_status)) return;
    for (int mt = warp; mt < d / 16; mt += NW + 1) {
      float c[NB][4];
      constexpr int KB = 4;  // k-steps whose fragments are loaded together
#pragma unroll
      for (int k0 = 0; k0 < NMV; k0 += KB) {
        uint32_t af[KB][4];
        float2 bx[KB], by[KB];
#pragma unroll
        for (int u = 0; u < KB; ++u)
          if (k0 + u < nmv) {
            const PieceLoc pl = locate(rV, d, 2 * (k0 + u) + a_chunk(lane));
            ldsm_x4(smem_u32(pmat) + swz(pl, 16 * mt + a_row(lane)), af[u]);
            const uint32_t xa = bfrag_addr(qt, xs, k0 + u, lane, NB);
            bx[u] = lds_f32x2(xa);
            by[u] = lds_f32x2(xa + 32u);
          }
#pragma unroll
        for (int u = 0; u < KB; ++u)
          if (k0 + u < nmv) {
            uint32_t bf[NB][2];
            bfrag_from<NB>(bx[u], by[u], lane, bf);
#pragma unroll
            for (int j = 0; j < NB; ++j) {
              if (k0 + u == 0) mma_bf16_z(c[j], af[u], bf[j][0], bf[j][1]);
              else mma_bf16(c[j], af[u], bf[j][0], bf[j][1]);
            }
          }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float o = NB == 1 ? c[0][e] + __shfl_xor_sync(kFull, c[0][e], 2) : c[0][e] + c[NB - 1][e];
        const int head = hA + (e & 1), i = 16 * mt + (lane >> 2) + 8 * (e >> 1);
        if (!lo_lane && head < nheads)
          a.out[((size_t)b * a.Hq + h0 + hbase + head * hstride) * d + i] = f32_to_bf16_rn(o);
      }
    }
  };
  if (S == 1) {  // this CTA finishes the unit alone: qt holds the normalised o~
    if (LAT) {
      for (int i = tid; i < gcount * rV; i += NT) {
        const int h = i / rV, j = i - h * rV;
        a.out[((size_t)b * a.Hq + h0 + h) * rV + j] = f32_to_bf16_rn(qt[h * xs + j]);
      }
    } else if (ok) {
      up_project(gcount, 0, 1);
    }
    return;
  }
  if (tagged_merge) {
    // ---- split merge through tagged words (no fence, no ticket) ------------------------
    // Every split has published its record (o~ scaled to its maximum, m, l) as tagged words;
    // the CTA of split s merges heads s, s + S, ...: it reads the records of its heads from
    // all splits (each word again until its tag says it was written; the whole grid is on
    // the GPU at once, so every split gets to publish), merges them, up-projects and writes
    // the output, and zeroes the words it read for the next call.
    if (s_idx >= gcount) {
      // P_V is only used by the merging CTAs, but its copy must land before this CTA's shared
      // memory is released (it was requested long before; the wait is bounded)
      if (!LAT && setup_ok && tid == 0) mbar_wait_bounded(setup_bar, 1u, a.dev_status);
      return;
    }
    const int nh = (gcount - s_idx + S - 1) / S;  // heads s_idx + hh S, hh < nh
    const int RP = RW / 2;                        // 16-byte word pairs per record
    const int SP = (S + 3) & ~3;                  // splits padded to whole float4s
    // The records' values, split-major per column: stg[(hh * RW + col) * SP + sp], so that a
    // column's splits are contiguous (float4 loads); splits [S, SP) hold m = -inf, l = o = 0.
    const uint32_t stgb = smem_u32(smem + L.region);
    const uint64_t* ubase = a.ws_words + (size_t)unit * S * G_T * RW;
    const int items = nh * S * RP;  // (record hh * S + sp, word pair)
    for (int i = tid; i < nh * RW * (SP - S); i += NT) {
      const int col = i / (SP - S), hh = col / RW;
      sts_f32(stgb + 4u * (uint32_t)(col * SP + S + (i - col * (SP - S))),
              col - hh * RW == rV ? -INFINITY : 0.f);
    }
    // A thread's items are tid, tid + NT, ...: their (hh, sp, pair) advance by fixed steps,
    // so no item needs a division.
    const int q_rec = NT / RP, q_pr = NT - q_rec * RP;
    int c_pr, c_sp, c_hh;
    auto first_item = [&]() {
      c_pr = tid % RP;
      const int rec = tid / RP;
      c_hh = rec / S;
      c_sp = rec - c_hh * S;
    };
    auto next_item = [&]() {
      c_pr += q_pr;
      int inc = q_rec;
      if (c_pr >= RP) {
        c_pr -= RP;
        ++inc;
      }
      c_sp += inc;
      while (c_sp >= S) {
        c_sp -= S;
        ++c_hh;
      }
    };
    auto item_src = [&]() {
      return ubase + ((size_t)c_sp * G_T + s_idx + c_hh * S) * RW + 2 * c_pr;
    };
    uint64_t t_wait = 0;  // when this thread first found a word not yet written
    bool gave_up = false;
    constexpr int kLd = 4;  // word pairs in flight per thread
    first_item();
    for (int i0 = tid; i0 < items; i0 += kLd * NT) {
      uint64_t w0[kLd], w1[kLd];
      const uint64_t* src[kLd];
      uint32_t dst[kLd];
#pragma unroll
      for (int u = 0; u < kLd; ++u) {
        if (i0 + u * NT < items) {
          src[u] = item_src();
          dst[u] = stgb + 4u * (uint32_t)((c_hh * RW + 2 * c_pr) * SP + c_sp);
          ld_tagged2(src[u], w0[u], w1[u]);
        }
        next_item();
      }
#pragma unroll
      for (int u = 0; u < kLd; ++u) {
        if (i0 + u * NT >= items) continue;
        while ((tagged_tag(w0[u]) & tagged_tag(w1[u])) != 1u && !gave_up) {
          const uint64_t now = global_timer_ns();
          if (t_wait == 0) {
            t_wait = now;
          } else if (now - t_wait > kWaitLimitNs) {
            report(a.dev_status, STIEF_DEV_WAIT_TIMEOUT);
            gave_up = true;
          }
          ld_tagged2(src[u], w0[u], w1[u]);
        }
        sts_f32(dst[u], tagged_value(w0[u]));
        sts_f32(dst[u] + 4u * (uint32_t)SP, tagged_value(w1[u]));
      }
    }
    __syncthreads();
    // the words read are in shared memory now: zero them for the next call (these stores
    // drain while the merge below runs)
    first_item();
    for (int i = tid; i < items; i += NT) {
      st_tagged2(const_cast<uint64_t*>(item_src()), 0ull, 0ull);
      next_item();
    }
    // merged, normalised o~ of head s_idx + hh S, column c: each thread forms the splits'
    // maximum and weights itself, into row hh of qt
    const uint32_t qtb = smem_u32(qt);
    for (int t = tid; t < nh * rV; t += NT) {
      const int hh = t / rV, c = t - hh * rV;
      const uint32_t mrow = stgb + 4u * (uint32_t)((hh * RW + rV) * SP);
      const uint32_t lrow = mrow + 4u * (uint32_t)SP, crow = stgb + 4u * (uint32_t)((hh * RW + c) * SP);
      float M = -INFINITY;
#pragma unroll 4
      for (int s4 = 0; s4 < SP; s4 += 4) {
        const float4 m4 = lds128f(mrow + 4u * (uint32_t)s4);
        M = fmaxf(M, fmaxf(fmaxf(m4.x, m4.y), fmaxf(m4.z, m4.w)));
      }
      float o = 0.f, Ls = 0.f;
      auto wgt = [&](float m) { return m == -INFINITY ? 0.f : ex2(m - M); };  // 0: no token
#pragma unroll 4
      for (int s4 = 0; s4 < SP; s4 += 4) {
        const uint32_t off = 4u * (uint32_t)s4;
        const float4 m4 = lds128f(mrow + off), l4 = lds128f(lrow + off), v4 = lds128f(crow + off);
        const float w0 = wgt(m4.x), w1 = wgt(m4.y), w2 = wgt(m4.z), w3 = wgt(m4.w);
        o = fmaf(w0, v4.x, fmaf(w1, v4.y, fmaf(w2, v4.z, fmaf(w3, v4.w, o))));
        Ls = fmaf(w0, l4.x, fmaf(w1, l4.y, fmaf(w2, l4.z, fmaf(w3, l4.w, Ls))));
      }
      sts_f32(qtb + 4u * (uint32_t)(hh * xs + c), Ls > 0.f ? o / Ls : 0.f);
    }
    __syncthreads();
    if (LAT) {  // o~ is the result
      for (int i = tid; i < nh * rV; i += NT) {
        const int hh = i / rV, j = i - hh * rV;
        a.out[((size_t)b * a.Hq + h0 + s_idx + hh * S) * rV + j] =
            f32_to_bf16_rn(lds_f32(qtb + 4u * (uint32_t)(hh * xs + j)));
      }
    } else {
      up_project(nh, s_idx, S);  // MMA columns 0 .. nh-1 carry the merged heads
    }
    return;
  }
  // Split partial states stay in the latent space (o~ scaled to the CTA's maximum, r_V floats
  // per head, then m and l): the last CTA merges them and up-projects once.
  const int rec = rV + 4;  // floats per partial state
  float* parts = a.ws_part + unit * (size_t)S * G_T * rec;
  for (int i = tid; i < gcount * rV; i += NT) {
    const int h = i / rV, j = i - h * rV;
    parts[((size_t)s_idx * G_T + h) * rec + j] = qt[h * xs + j];
  }

  // ---- split merge: publish this split, take a ticket; the last CTA merges them all ---------
  if (tid < gcount) {
    parts[((size_t)s_idx * G_T + tid) * rec + rV] = fin[tid];
    parts[((size_t)s_idx * G_T + tid) * rec + rV + 1] = fin[8 + tid];
  }
  __syncthreads();  // every state of this CTA is written (block scope) ...
  if (tid == 0) {
    // ... and the acquire-release ticket makes them, by cumulativity, visible device-wide
    // before the count moves; the last CTA's acquire orders its reads of the others' states
    uint32_t ticket;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;"
                 : "=r"(ticket)
                 : "l"(a.ws_cnt + unit)
                 : "memory");
    const int last = ticket == (uint32_t)(S - 1);
    if (last) a.ws_cnt[unit] = 0u;  // ready for the next call
    *flag = last;
  }
  __syncthreads();
  if (!*flag) {
    // P_V is only used by the merging CTA, but its copy must land before this CTA's shared
    // memory is released (it was requested long before; the wait is bounded)
    if (!LAT && setup_ok && tid == 0) mbar_wait_bounded(setup_bar, 1u, a.dev_status);
    return;
  }
  // Thread groups of tpi consecutive lanes take one item = (head, 4 output columns); lane
  // `sub` of a group merges splits sub, sub + tpi, ... (a batch of eight in flight at a time),
  // then the group combines its tpi running states with shuffles.
  const int nitems = gcount * (rV / 4);
  int tpi = 1;
  while (tpi < 8 && tpi * 2 * nitems <= NT) tpi *= 2;
  const int sub = tid & (tpi - 1);
  const int iters = (nitems * tpi + NT - 1) / NT;
  auto merge = [](float& M, float& Ls, float4& o, float m2, float l2, const float4& o2) {
    if (m2 == -INFINITY) return;
    if (m2 > M) {
      const float f = ex2(M - m2);  // 0 while M is -inf
      Ls *= f;
      o.x *= f;
      o.y *= f;
      o.z *= f;
      o.w *= f;
      M = m2;
    }
    const float w = ex2(m2 - M);
    Ls = fmaf(w, l2, Ls);
    o.x = fmaf(w, o2.x, o.x);
    o.y = fmaf(w, o2.y, o.y);
    o.z = fmaf(w, o2.z, o.z);
    o.w = fmaf(w, o2.w, o.w);
  };
  constexpr int kBatch = 8;
  for (int it = 0; it < iters; ++it) {
    const int item = (it * NT + tid) / tpi;
    const bool valid = item < nitems;
    const int g = valid ? item / (rV / 4) : 0, c4 = valid ? item - g * (rV / 4) : 0;
    float M = -INFINITY, Ls = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = sub; s0 < S; s0 += kBatch * tpi) {
      float ms[kBatch], ls[kBatch];
      float4 os[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int s = s0 + u * tpi;
        if (valid && s < S) {
          const float* r = parts + ((size_t)s * G_T + g) * rec;
          const float2 m2 = __ldcg(reinterpret_cast<const float2*>(r + rV));
          ms[u] = m2.x;
          ls[u] = m2.y;
          os[u] = __ldcg(reinterpret_cast<const float4*>(r) + c4);
        } else {
          ms[u] = -INFINITY;
          ls[u] = 0.f;
          os[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      // the batch's maximum first, then independent weights and sums (short dependency chains)
      float Mb = -INFINITY;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) Mb = fmaxf(Mb, ms[u]);
      float Lb2 = 0.f;
      float4 ob = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const float w = ms[u] == -INFINITY ? 0.f : ex2(ms[u] - Mb);
        Lb2 = fmaf(w, ls[u], Lb2);
        ob.x = fmaf(w, os[u].x, ob.x);
        ob.y = fmaf(w, os[u].y, ob.y);
        ob.z = fmaf(w, os[u].z, ob.z);
        ob.w = fmaf(w, os[u].w, ob.w);
      }
      merge(M, Ls, o, Mb, Lb2, ob);
    }
    for (int off = 1; off < tpi; off <<= 1) {
      const float M2 = __shfl_xor_sync(kFull, M, off), L2 = __shfl_xor_sync(kFull, Ls, off);
      float4 o2;
      o2.x = __shfl_xor_sync(kFull, o.x, off);
      o2.y = __shfl_xor_sync(kFull, o.y, off);
      o2.z = __shfl_xor_sync(kFull, o.z, off);
      o2.w = __shfl_xor_sync(kFull, o.w, off);
      merge(M, Ls, o, M2, L2, o2);
    }
    if (valid && sub == 0) {
      const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
      if (LAT) {  // o~ is the result
        uint2 packed;
        packed.x = pack_bf16x2_rn(o.x * inv, o.y * inv);
        packed.y = pack_bf16x2_rn(o.z * inv, o.w * inv);
        *reinterpret_cast<uint2*>(a.out + ((size_t)b * a.Hq + h0 + g) * rV + 4 * c4) = packed;
      } else {  // the normalised o~ becomes the up-projection's operand
        float* dst = qt + g * xs + 4 * c4;
        dst[0] = o.x * inv;
        dst[1] = o.y * inv;
        dst[2] = o.z * inv;
        dst[3] = o.w * inv;
      }
    }
  }
  if (!LAT) {
    __syncthreads();
    up_project(gcount, 0, 1);
  }
}

// ------------------------------------------------------------------------------ launch

template <int NB, int NKS, int NMV, int TT, int MODE>
static cudaError_t launch_k(const DecodeArgs& a, cudaStream_t stream) {
  const DecodeSmem L = decode_smem_layout(a.nwarps, a.nstage, a.rK, a.rV, TT,
                                          MODE == kModeQ8 || MODE == kModePagedQ8 || MODE == kModeQ8Append
                                              ? 1
                                              : MODE == kModeQ4 ? 2 : 0);
  auto kern = stief_decode_kernel<NB, NKS, NMV, TT, MODE>;
  static SmemLimit limit;
  cudaError_t e = limit.ensure(reinterpret_cast<const void*>(kern), a.device, (int)L.total);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.S, a.Hkv * a.qsub, a.B);
  cfg.blockDim = dim3((a.nwarps + 1) * 32);  // consumer warps + the producer warp
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  // programmatic dependent launch: the CTAs may be scheduled while the previous kernel in
  // the stream drains; they wait for it (griddepcontrol.wait) before reading any input
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

// The tile configurations of one mode: NB n-tiles (group tiles of up to 4 or 8 heads), the
// key / value rank bounds (64 or 128) and the tile (32 tokens, or 64 for small ranks).
template <int MODE, int NB>
static cudaError_t launch_mode_nb(const DecodeArgs& a, cudaStream_t stream) {
  const bool wk = a.rK > 64, wv = a.rV > 64;
  if (a.tile == 64) {  // only small ranks (both <= 64, rK + rV <= 96) take 64-token tiles
    if (wk || wv) return cudaErrorInvalidValue;
    return launch_k<NB, 4, 4, 64, MODE>(a, stream);
  }
  if (!wk && !wv) return launch_k<NB, 4, 4, 32, MODE>(a, stream);
  if (!wk) return launch_k<NB, 4, 8, 32, MODE>(a, stream);
  if (!wv) return launch_k<NB, 8, 4, 32, MODE>(a, stream);
  return launch_k<NB, 8, 8, 32, MODE>(a, stream);
}

template <int MODE>
static cudaError_t launch_mode(const DecodeArgs& a, cudaStream_t stream) {
  return a.G_T <= 4 ? launch_mode_nb<MODE, 1>(a, stream) : launch_mode_nb<MODE, 2>(a, stream);
}

// One translation unit per mode instantiates it (they compile side by side).
cudaError_t launch_decode_plain(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_latent(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_paged(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_q8(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_q8_append(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_q4(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_paged_q8(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_joint_v(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_latent_joint_v(const DecodeArgs& a, cudaStream_t stream);

}  // namespace stief
