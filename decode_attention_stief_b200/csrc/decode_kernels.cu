// decode_kernels.cu -- split-KV decode attention over the latent (Stiefel-projected)
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
// One kernel, stief_decode_kernel<G_T, NP>, grid (splits, Hkv * qsub, B).  A CTA
// serves up to G_T query heads of one KV head ("unit") over one token range, with
// NP warp pairs (2*NP warps):
//   - prologue: q and P_K[h] arrive by bulk copy; q~ = q . P_K * log2(e)/sqrt(d)
//     in fp32, stored padded chunk-major
//   - streaming: pair i owns two rings of shared-memory stages holding the keys
//     and the values of 32-token tiles, each slot filled by a 1-D bulk copy (TMA
//     engine, L2 evict-first) that completes on the slot's mbarrier, and works
//     through tiles i, i + NP, ...  Its K-warp computes the scores -- one lane
//     per token; key tiles land by 2-D TMA tensor copies in 64/32/16-column pieces
//     with the matching 128/64/32-byte swizzle, so all lanes read the same logical
//     chunk at once without bank conflicts and q~ is read as warp-wide broadcasts;
//     packed fp32x2 FMAs -- and the online
//     softmax in the log2
//     domain with lazy rescaling (accumulators rescaled only when a score passes
//     the running reference by more than 8, so every weight stays <= 2^8).  It
//     hands the weights (as duplicated pairs) and any rescale factors to its
//     V-warp through a double buffer guarded by two mbarriers.  The V-warp mixes
//     the latent values (r_V/8 lanes per token, packed FMAs).  Key and value halves
//     of a tile live in separate rings, each refilled by its own consumer as soon
//     as it is done, which keeps more bytes in flight.  Splitting the roles halves the registers each warp needs, so twice
//     as many warps hide shared-memory and FMA latency.  No CTA-wide barrier in
//     the loop.
//   - epilogue: merge the pairs; with one split the CTA finishes the unit itself;
//     otherwise it stores its partial state (o~[r_V], m, l) and takes a ticket,
//     and the last CTA of the unit merges all splits (log-sum-exp) -- that CTA
//     resets the ticket counter, so the workspace counters stay zero between
//     calls.  P_V arrives by bulk copy into the freed stage region while the
//     merge runs; then o = o~ . P_V^T, bf16 out.
#include <cfloat>
#include <cmath>
#include <cstdint>

#include "stief_device.cuh"
#include "stief_internal.h"

namespace stief {

constexpr int kTile = 32;            // tokens per pair tile
constexpr float kRescaleTau = 8.0f;  // lazy-rescale threshold (log2 units)

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float2 f2(float x, float y) { return make_float2(x, y); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
// the 4 bf16 pairs of a 16-byte chunk, widened exactly to fp32 pairs
__device__ __forceinline__ void unpack8(const uint4 w, float2 (&v)[4]) {
  v[0] = f2(bf16lo(w.x), bf16hi(w.x));
  v[1] = f2(bf16lo(w.y), bf16hi(w.y));
  v[2] = f2(bf16lo(w.z), bf16hi(w.z));
  v[3] = f2(bf16lo(w.w), bf16hi(w.w));
}

__device__ __forceinline__ float4 ldcg4(const float* p) {
  return __ldcg(reinterpret_cast<const float4*>(p));
}

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// Shared-memory carve-up (byte offsets from the dynamic base).
struct DecodeSmem {
  uint32_t bars;     // NP*ns K-stage, NP*ns V-stage, NP*2 weights-full, NP*2 weights-empty, 1 setup
  uint32_t q;        // G_T x d bf16 query rows
  uint32_t qt;       // (rK/8) chunks x G_T x 8 fp32 projected, scaled queries
  uint32_t fbuf;     // NP x 2 x (G_T factors + flag): rescale handed from K- to V-warp
  uint32_t ml;       // NP x G_T x (m, l); then G_T x (M, L, rescale); then a flag
  uint32_t scratch;  // P_K (prologue); NP x 2 x 32 x G_T x 2 fp32 weights; o~ (epilogue)
  uint32_t region;   // per pair a K ring then a V ring of stages; later reduction /
                     // split-merge staging + P_V at its end
  uint32_t region_bytes;
  uint32_t pv;       // offset of P_V inside the region (epilogue)
  uint32_t total;
};

__host__ __device__ inline DecodeSmem decode_smem_layout(int NP, int nstage, int G_T, int d, int rK,
                                                         int rV) {
  DecodeSmem s;
  uint32_t off = 0;
  s.bars = off;
  off = align_up(off + 8u * (2 * NP * nstage + 4 * NP + 1), 128);
  s.q = off;
  off = align_up(off + 2u * G_T * d, 128);
  s.qt = off;
  off = align_up(off + 4u * rK * G_T, 128);
  s.fbuf = off;
  off = align_up(off + 4u * NP * 2 * (G_T + 1), 128);
  s.ml = off;
  off = align_up(off + 4u * (2 * NP * G_T + 3 * G_T + 4), 128);
  s.scratch = off;
  const uint32_t pbuf = 8u * NP * 2 * kTile * G_T;
  const uint32_t pk = 2u * d * rK;
  const uint32_t ob = 4u * G_T * rV;
  uint32_t sb = pbuf > pk ? pbuf : pk;
  sb = sb > ob ? sb : ob;
  off = align_up(off + sb, 128);
  off = align_up(off, 1024);  // swizzled key slots need 1 KiB alignment
  s.region = off;
  const uint32_t stage = (uint32_t)NP * nstage * kTile * (rK + rV) * 2u;
  const uint32_t red = (uint32_t)NP * 32u * G_T * 8u * 4u;
  const uint32_t pvb = align_up(2u * d * rV, 128);
  const uint32_t need = align_up(red, 128) + pvb;
  s.region_bytes = align_up(stage > need ? stage : need, 128);
  s.pv = s.region_bytes - pvb;
  off += s.region_bytes;
  s.total = off;
  return s;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Scores of one key piece for the lane's token: WC 16-byte chunks per row, stored
// swizzled (chunk c of the lane's row at byte (c << 4) ^ sw4 of the row); q~ chunks are
// warp-wide broadcasts.  prow_sw = row address ^ sw4 (rows are at least 32-byte aligned
// and the swizzle only touches bits below the row size, so XOR equals addition).
template <int G_T, int WC>
__device__ __forceinline__ void score_piece(uint32_t prow_sw, uint32_t q0, float2 (&sa)[G_T],
                                            float2 (&sb)[G_T]) {
  constexpr uint32_t QS = (uint32_t)G_T * 32u;  // bytes per q~ chunk row
#pragma unroll
  for (int cc = 0; cc < WC; cc += 2) {
    float2 ka[4], kb[4];
    unpack8(lds128(prow_sw ^ (uint32_t)(cc << 4)), ka);
    unpack8(lds128(prow_sw ^ (uint32_t)((cc + 1) << 4)), kb);
    const uint32_t qa = q0 + (uint32_t)cc * QS;
#pragma unroll
    for (int g = 0; g < G_T; ++g) {
      const float4 xa = lds128f(qa + g * 32u), ya = lds128f(qa + g * 32u + 16u);
      const float4 xb = lds128f(qa + QS + g * 32u), yb = lds128f(qa + QS + g * 32u + 16u);
      sa[g] = fma2(f2(xa.x, xa.y), ka[0], sa[g]);
      sb[g] = fma2(f2(xb.x, xb.y), kb[0], sb[g]);
      sa[g] = fma2(f2(xa.z, xa.w), ka[1], sa[g]);
      sb[g] = fma2(f2(xb.z, xb.w), kb[1], sb[g]);
      sa[g] = fma2(f2(ya.x, ya.y), ka[2], sa[g]);
      sb[g] = fma2(f2(yb.x, yb.y), kb[2], sb[g]);
      sa[g] = fma2(f2(ya.z, ya.w), ka[3], sa[g]);
      sb[g] = fma2(f2(yb.z, yb.w), kb[3], sb[g]);
    }
  }
}

// Latent value mix of one tile: RVC = rV/8 lanes per token, TPW tokens per step; the
// lane's token slot and chunk are fixed, so every address is a constant offset.
template <int G_T, int RVC>
__device__ __forceinline__ void mix_tile(uint32_t vst, uint32_t p_addr, int n, int lane,
                                         float2 (&acc)[G_T][4]) {
  constexpr int TPW = 32 / RVC;
  constexpr int STEPS = (32 + TPW - 1) / TPW;
  const int vslot = lane / RVC;
  if (vslot >= TPW) return;
  const int vchunk = lane - vslot * RVC;
  const uint32_t vb = vst + (uint32_t)(vslot * RVC + vchunk) * 16u;
  const uint32_t pb = p_addr + (uint32_t)vslot * G_T * 8u;
#pragma unroll
  for (int st = 0; st < STEPS; ++st) {
    if (st * TPW + vslot < n) {
      float2 v[4];
      unpack8(lds128(vb + (uint32_t)(st * TPW * RVC * 16)), v);
      float2 pp[G_T];
      if constexpr (G_T >= 2) {
#pragma unroll
        for (int g2 = 0; g2 < G_T; g2 += 2) {
          const float4 x = lds128f(pb + (uint32_t)(st * TPW * G_T * 8 + g2 * 8));
          pp[g2] = f2(x.x, x.y);
          pp[g2 + 1] = f2(x.z, x.w);
        }
      } else {
        pp[0] = *reinterpret_cast<const float2*>(
            __cvta_shared_to_generic(pb + (uint32_t)(st * TPW * 8)));
      }
#pragma unroll
      for (int g = 0; g < G_T; ++g)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[g][e] = fma2(pp[g], v[e], acc[g][e]);
    }
  }
}

// Warp-specialised: warps [0, NP) are K-warps (scores, softmax), warps [NP, 2NP) are
// V-warps (value mix, stage refills).  K-warp i and V-warp i form pair i, which owns a
// ring of `nstage` stages and processes the CTA's tiles i, i + NP, i + 2NP, ...
template <int G_T, int NP>
__global__ void __launch_bounds__(NP * 64, 1) stief_decode_kernel(const __grid_constant__ DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int NT = NP * 64;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const bool is_k = warp < NP;
  const int pair = is_k ? warp : warp - NP;
  const int s_idx = blockIdx.x;                 // split
  const int kvh = blockIdx.y / a.qsub;          // KV head
  const int qs = blockIdx.y - kvh * a.qsub;     // query sub-group of that head
  const int b = blockIdx.z;
  const int d = a.d, rK = a.rK, rV = a.rV, S = a.S;
  const int ns = a.nstage;
  const int h0 = kvh * a.G + qs * G_T;          // first query head of this CTA
  const int gcount = min(G_T, a.G - qs * G_T);  // valid query heads here
  const size_t unit = ((size_t)b * a.Hkv + kvh) * a.qsub + qs;

  const DecodeSmem L = decode_smem_layout(NP, ns, G_T, d, rK, rV);
  uint64_t* kfull = reinterpret_cast<uint64_t*>(smem + L.bars);  // [NP][ns]
  uint64_t* vfull = kfull + NP * ns;                              // [NP][ns]
  uint64_t* pfull = vfull + NP * ns;                              // [NP][2]
  uint64_t* pempty = pfull + NP * 2;                             // [NP][2]
  uint64_t* setup_bar = pempty + NP * 2;  // phase 0: q + P_K, phase 1: P_V
  // a key slot holds the tile's column pieces (64/32/16 wide) as the TMA engine writes
  // them, each with its shared-memory swizzle; a value slot holds the rows unchanged
  const uint32_t kt_bytes = (uint32_t)kTile * rK * 2u, vt_bytes = (uint32_t)kTile * rV * 2u;
  uint8_t* my_kring = smem + L.region + (size_t)pair * ns * (kt_bytes + vt_bytes);
  uint8_t* my_vring = my_kring + (size_t)ns * kt_bytes;
  float* ml = reinterpret_cast<float*>(smem + L.ml);
  float* fin = ml + 2 * NP * G_T;                    // [G_T] M, [G_T] L, [G_T] rescale
  int* flag = reinterpret_cast<int*>(fin + 3 * G_T);
  float* fbuf = reinterpret_cast<float*>(smem + L.fbuf) + pair * 2 * (G_T + 1);

  if ((smem_u32(smem + L.region) & 1023u) != 0) {  // swizzle patterns assume 1 KiB alignment
    if (tid == 0) report(a.dev_status, STIEF_DEV_SMEM_ALIGN);
    return;
  }
  if (tid == 0) {
    for (int i = 0; i < 2 * NP * ns + 4 * NP + 1; ++i) mbar_init(&kfull[i], 1);
    fence_barrier_init();
  }
  __syncthreads();

  // q and the bases were written before this kernel started (it is not launched
  // as a programmatic dependent), so they may be fetched before the wait below.
  if (tid == 0) {
    const uint32_t qbytes = 2u * gcount * d;
    const uint32_t pbytes = 2u * d * rK;
    mbar_arrive_expect_tx(setup_bar, qbytes + pbytes);
    bulk_g2s(smem + L.q, a.q + ((size_t)b * a.Hq + h0) * d, qbytes, setup_bar);
    bulk_g2s(smem + L.scratch, a.P_K + (size_t)kvh * d * rK, pbytes, setup_bar);
  }
  pdl_wait();

  int Lb = a.seq_lens[b];
  if (Lb < 0 || Lb > a.L_max) {
    if (tid == 0 && s_idx == 0 && blockIdx.y == 0) report(a.dev_status, STIEF_DEV_BAD_LENGTH);
    Lb = 0;
  }
  const int chunk = (Lb + S - 1) / S;
  const int t0 = min(Lb, s_idx * chunk);
  const int t1 = min(Lb, t0 + chunk);
  const int n_tiles = (t1 - t0 + kTile - 1) / kTile;
  const int my_tiles = pair < n_tiles ? (n_tiles - pair + NP - 1) / NP : 0;

  const size_t head_row0 = ((size_t)b * a.Hkv + kvh) * a.L_max;
  const uint16_t* vbase_g = a.v_lat + head_row0 * rV;

  // K and V halves of a tile travel separately, so each ring slot is refilled as soon
  // as its own consumer is done with it (the K-warp after its scores, the V-warp
  // after its mix): more bytes stay in flight per SM.
  // K and V halves of a tile travel separately, so each ring slot is refilled as soon
  // as its own consumer is done with it (the K-warp after its scores, the V-warp
  // after its mix).  Keys arrive by 2-D TMA tensor copies (swizzled), values by
  // one 1-D bulk copy.
  auto issue_k = [&](int k, uint64_t policy) {  // lane 0 of the K-warp
    const int tok0 = t0 + (pair + k * NP) * kTile;
    uint8_t* dst = my_kring + (size_t)(k % ns) * kt_bytes;
    uint64_t* bar = &kfull[pair * ns + (k % ns)];
    // whole 32-row boxes land (rows past the tile are masked out of the softmax)
    mbar_arrive_expect_tx(bar, kt_bytes);
    const int y = (int)(head_row0 + tok0);
    for (int p = 0; p < a.npieces; ++p)
      tma_load_2d(dst + a.kp[p].smem_off, &a.tmk[a.kp[p].map], a.kp[p].x, y, bar, policy);
  };
  auto issue_v = [&](int k, uint64_t policy) {  // lane 0 of the V-warp
    const int tok0 = t0 + (pair + k * NP) * kTile;
    const int n = min(kTile, t1 - tok0);
    uint64_t* bar = &vfull[pair * ns + (k % ns)];
    const uint32_t bytes = (uint32_t)n * rV * 2u;
    mbar_arrive_expect_tx(bar, bytes);
    bulk_g2s_hint(my_vring + (size_t)(k % ns) * vt_bytes, vbase_g + (size_t)tok0 * rV, bytes, bar,
                  policy);
  };
  int issued = min(ns, my_tiles);  // tiles this warp has requested
  {
    const uint64_t policy = l2_policy_evict_first();
    if (lane == 0)
      for (int k = 0; k < issued; ++k) {
        if (is_k) issue_k(k, policy);
        else issue_v(k, policy);
      }
  }

  // ---- q~ = q . P_K, scaled into the log2 domain -----------------------------------
  // thread = (query head g, column pair cp, half of d); the two halves of a pair sit in
  // adjacent lanes and are added with one shuffle.
  bool ok = mbar_wait_bounded(setup_bar, 0, a.dev_status);
  {
    const int qstride = G_T * 8;  // floats per chunk row
    const uint32_t* q2 = reinterpret_cast<const uint32_t*>(smem + L.q);
    const uint32_t* pk2 = reinterpret_cast<const uint32_t*>(smem + L.scratch);
    float* qt = reinterpret_cast<float*>(smem + L.qt);
    const int half = rK / 2;  // column pairs
    const int outs = G_T * half;
    const int parts = NT >= 2 * outs ? 2 : 1;
    const int total = outs * parts;
    const int total_r = (total + 31) & ~31;  // whole warps take part in the shuffle
    const int span = (d / 2) / parts;
    for (int idx = tid; idx < total_r; idx += NT) {
      const bool act = idx < total;
      const int o = idx / parts, part = idx - o * parts;
      const int g = o / half, cp = o - g * half;
      float2 acc = f2(0.f, 0.f);
      if (act && ok && g < gcount) {
        const uint32_t* qrow = q2 + g * (d / 2);
#pragma unroll 4
        for (int i2 = part * span; i2 < (part + 1) * span; ++i2) {
          const uint32_t qq = qrow[i2];  // q[2*i2], q[2*i2+1]
          const uint32_t pa = pk2[(2 * i2) * half + cp];
          const uint32_t pb = pk2[(2 * i2 + 1) * half + cp];
          const float q0 = bf16lo(qq), q1 = bf16hi(qq);
          acc = fma2(f2(q0, q0), f2(bf16lo(pa), bf16hi(pa)), acc);
          acc = fma2(f2(q1, q1), f2(bf16lo(pb), bf16hi(pb)), acc);
        }
      }
      if (parts == 2) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 1);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 1);
      }
      if (act && part == 0) {
        const int c = 2 * cp;
        float* dst = qt + (c >> 3) * qstride + g * 8 + (c & 7);
        dst[0] = acc.x * a.qscale;
        dst[1] = acc.y * a.qscale;
      }
    }
  }
  __syncthreads();

  // ---- streaming ------------------------------------------------------------------------
  const int RV = rV >> 3;
  const int TPW = 32 / RV;            // tokens per value step
  const int vslot = lane / RV;
  const bool vactive = vslot < TPW;
  float* pbuf = reinterpret_cast<float*>(smem + L.scratch) + pair * 2 * kTile * G_T * 2;

  float m_ref[G_T], l_lane[G_T];
  float2 acc[G_T][4];
#pragma unroll
  for (int g = 0; g < G_T; ++g) {
    m_ref[g] = -INFINITY;
    l_lane[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[g][e] = f2(0.f, 0.f);
  }
  int consumed = 0;

  if (is_k) {
    const uint32_t qstride_b = (uint32_t)G_T * 32u;
    const uint32_t qt_addr = smem_u32(smem + L.qt);
    const uint64_t policy = l2_policy_evict_first();
    for (int k = 0; k < my_tiles && ok; ++k) {
      const int stg = k % ns;
      if (!mbar_wait_bounded(&kfull[pair * ns + stg], (uint32_t)((k / ns) & 1), a.dev_status)) {
        ok = false;
        break;
      }
      const int tok0 = t0 + (pair + k * NP) * kTile;
      const int n = min(kTile, t1 - tok0);
      const uint32_t kst = smem_u32(my_kring + (size_t)stg * kt_bytes);

      // scores: lane = token; two chunks per iteration (RK is even); q~ chunk reads are
      // warp-wide broadcasts
      float s[G_T];
      {
        float2 sa[G_T], sb[G_T];
#pragma unroll
        for (int g = 0; g < G_T; ++g) {
          sa[g] = f2(0.f, 0.f);
          sb[g] = f2(0.f, 0.f);
        }
        for (int p = 0; p < a.npieces; ++p) {
          const int w = a.kp[p].width;
          const uint32_t prow = kst + (uint32_t)a.kp[p].smem_off + (uint32_t)lane * w * 2u;
          const uint32_t q0 = qt_addr + (uint32_t)(a.kp[p].x >> 3) * qstride_b;
          if (w == 64) score_piece<G_T, 8>(prow ^ ((uint32_t)(lane & 7) << 4), q0, sa, sb);
          else if (w == 32) score_piece<G_T, 4>(prow ^ ((uint32_t)((lane >> 1) & 3) << 4), q0, sa, sb);
          else score_piece<G_T, 2>(prow ^ ((uint32_t)((lane >> 2) & 1) << 4), q0, sa, sb);
        }
#pragma unroll
        for (int g = 0; g < G_T; ++g) s[g] = (sa[g].x + sa[g].y) + (sb[g].x + sb[g].y);
      }
      // the key slot is free: request the keys of tile k + ns
      __syncwarp();
      consumed = k + 1;
      if (k + ns < my_tiles) {
        if (lane == 0) issue_k(k + ns, policy);
        issued = k + ns + 1;
      }

      // online softmax (log2 domain), lazy rescale; factors go to the V-warp
      const bool valid = lane < n;
      float pw[G_T], fac[G_T];
      bool rescaled = false;
#pragma unroll
      for (int g = 0; g < G_T; ++g) {
        const float sg = valid ? s[g] : -INFINITY;
        fac[g] = 1.f;
        if (__any_sync(0xffffffffu, sg > m_ref[g] + kRescaleTau)) {
          const float m_new = fmaxf(m_ref[g], warp_max(sg));
          fac[g] = ex2(m_ref[g] - m_new);  // 0 when m_ref was -inf
          l_lane[g] *= fac[g];
          m_ref[g] = m_new;
          rescaled = true;
        }
        pw[g] = valid ? ex2(sg - m_ref[g]) : 0.f;
        l_lane[g] += pw[g];
      }
      const int pb = k & 1;
      if (k >= 2 && !mbar_wait_bounded(&pempty[pair * 2 + pb], (uint32_t)(((k >> 1) - 1) & 1),
                                       a.dev_status)) {
        ok = false;
        break;
      }
      float* pt = pbuf + pb * kTile * G_T * 2;
      if constexpr (G_T >= 2) {
#pragma unroll
        for (int g2 = 0; g2 < G_T; g2 += 2)
          *reinterpret_cast<float4*>(pt + (lane * G_T + g2) * 2) =
              make_float4(pw[g2], pw[g2], pw[g2 + 1], pw[g2 + 1]);
      } else {
        *reinterpret_cast<float2*>(pt + lane * 2) = f2(pw[0], pw[0]);
      }
      if (lane == 0) {
        float* fb = fbuf + pb * (G_T + 1);
#pragma unroll
        for (int g = 0; g < G_T; ++g) fb[g] = fac[g];
        fb[G_T] = rescaled ? 1.f : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&pfull[pair * 2 + pb]);
    }
  } else {
    const uint64_t policy = l2_policy_evict_first();
    for (int k = 0; k < my_tiles && ok; ++k) {
      const int pb = k & 1;
      if (!mbar_wait_bounded(&pfull[pair * 2 + pb], (uint32_t)((k >> 1) & 1), a.dev_status) ||
          !mbar_wait_bounded(&vfull[pair * ns + (k % ns)], (uint32_t)((k / ns) & 1), a.dev_status)) {
        ok = false;
        break;
      }
      const int tok0 = t0 + (pair + k * NP) * kTile;
      const int n = min(kTile, t1 - tok0);
      const uint32_t vst = smem_u32(my_vring + (size_t)(k % ns) * vt_bytes);
      const float* fb = fbuf + pb * (G_T + 1);
      if (fb[G_T] != 0.f) {
#pragma unroll
        for (int g = 0; g < G_T; ++g) {
          const float f = fb[g];
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[g][e] = f2(acc[g][e].x * f, acc[g][e].y * f);
        }
      }
      const uint32_t p_addr = smem_u32(pbuf + pb * kTile * G_T * 2);
      switch (RV) {
        case 2: mix_tile<G_T, 2>(vst, p_addr, n, lane, acc); break;
        case 4: mix_tile<G_T, 4>(vst, p_addr, n, lane, acc); break;
        case 6: mix_tile<G_T, 6>(vst, p_addr, n, lane, acc); break;
        case 8: mix_tile<G_T, 8>(vst, p_addr, n, lane, acc); break;
        case 10: mix_tile<G_T, 10>(vst, p_addr, n, lane, acc); break;
        case 12: mix_tile<G_T, 12>(vst, p_addr, n, lane, acc); break;
        case 14: mix_tile<G_T, 14>(vst, p_addr, n, lane, acc); break;
        default: mix_tile<G_T, 16>(vst, p_addr, n, lane, acc); break;
      }
      __syncwarp();
      consumed = k + 1;
      if (lane == 0) {
        mbar_arrive(&pempty[pair * 2 + pb]);
        if (k + ns < my_tiles) {
          issue_v(k + ns, policy);
          issued = k + ns + 1;
        }
      }
    }
  }
  // copies that were requested but not consumed (only after a timed-out wait) must land
  // before the region is reused or the CTA exits
  if (lane == 0)
    for (int k = consumed; k < issued; ++k)
      mbar_wait_bounded(&(is_k ? kfull : vfull)[pair * ns + (k % ns)], (uint32_t)((k / ns) & 1),
                        nullptr);

  // ---- merge the pairs ---------------------------------------------------------------
  if (is_k) {
#pragma unroll
    for (int g = 0; g < G_T; ++g) {
      const float lw = warp_sum(l_lane[g]);
      if (lane == 0) {
        ml[(pair * G_T + g) * 2 + 0] = m_ref[g];
        ml[(pair * G_T + g) * 2 + 1] = lw;
      }
    }
  }
  __syncthreads();  // every pair is done with its stages: the region becomes the reduction buffer
  // P_V for the up-projection: needed here when this CTA finishes the unit itself
  if (tid == 0 && S == 1) {
    fence_proxy_async_smem();
    const uint32_t vbytes = 2u * d * rV;
    mbar_arrive_expect_tx(setup_bar, vbytes);
    bulk_g2s(smem + L.region + L.pv, a.P_V + (size_t)kvh * d * rV, vbytes, setup_bar);
  }
  float* red = reinterpret_cast<float*>(smem + L.region);
  if (!is_k) {
    float* mine = red + ((size_t)pair * 32 + lane) * G_T * 8;
#pragma unroll
    for (int g = 0; g < G_T; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        mine[g * 8 + 2 * e] = vactive ? acc[g][e].x : 0.f;
        mine[g * 8 + 2 * e + 1] = vactive ? acc[g][e].y : 0.f;
      }
  }
  __syncthreads();

  float* ot = reinterpret_cast<float*>(smem + L.scratch);  // o~ [G_T][rV] for the up-projection
  const int part_stride = rV + 4;
  float* parts = a.ws_part + unit * (size_t)S * G_T * part_stride;  // this unit's S x G_T states
  for (int idx = tid; idx < G_T * rV; idx += NT) {
    const int g = idx / rV, jj = idx - g * rV;
    const int c = jj >> 3, e = jj & 7;
    float M = -INFINITY;
    for (int w = 0; w < NP; ++w) M = fmaxf(M, ml[(w * G_T + g) * 2]);
    float o = 0.f, lsum = 0.f;
    for (int w = 0; w < NP; ++w) {
      const float mw = ml[(w * G_T + g) * 2];
      const float sc = (mw == -INFINITY) ? 0.f : ex2(mw - M);
      float part = 0.f;
      for (int slot = 0; slot < TPW; ++slot)
        part += red[((size_t)w * 32 + slot * RV + c) * G_T * 8 + g * 8 + e];
      o = fmaf(sc, part, o);
      lsum = fmaf(sc, ml[(w * G_T + g) * 2 + 1], lsum);
    }
    if (S == 1) {
      ot[g * rV + jj] = lsum > 0.f ? o / lsum : 0.f;
    } else {
      float* pdst = parts + ((size_t)s_idx * G_T + g) * part_stride;
      pdst[jj] = o;
      if (jj == 0) {
        pdst[rV] = M;
        pdst[rV + 1] = lsum;
      }
    }
  }

  if (S > 1) {
    // publish this split and take a ticket; the last CTA of the unit merges every split
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const uint32_t ticket = atomicAdd(a.ws_cnt + unit, 1u);
      const int last = ticket == (uint32_t)(S - 1);
      if (last) {
        a.ws_cnt[unit] = 0u;  // ready for the next call
        fence_proxy_async_smem();
        const uint32_t vbytes = 2u * d * rV;
        mbar_arrive_expect_tx(setup_bar, vbytes);
        bulk_g2s(smem + L.region + L.pv, a.P_V + (size_t)kvh * d * rV, vbytes, setup_bar);
      }
      *flag = last;
    }
    __syncthreads();
    if (!*flag) return;
    __threadfence();
    // stage the unit's split states through shared memory (below P_V), a chunk of splits
    // at a time, accumulating against a running maximum
    float* stage_p = reinterpret_cast<float*>(smem + L.region);
    const int per_split = G_T * part_stride;  // floats
    const int s_chunk = max(1, (int)(L.pv / 4u) / per_split);
    for (int s0 = 0; s0 < S; s0 += s_chunk) {
      const int nsp = min(s_chunk, S - s0);
      const int n4 = nsp * per_split / 4;
      const float* src = parts + (size_t)s0 * per_split;
      for (int i = tid; i < n4; i += NT * 4) {
        float4 x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (i + u * NT < n4) x[u] = ldcg4(src + 4 * (i + u * NT));
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (i + u * NT < n4) reinterpret_cast<float4*>(stage_p)[i + u * NT] = x[u];
      }
      __syncthreads();
      if (tid < G_T) {
        const float M_old = (s0 == 0) ? -INFINITY : fin[tid];
        float M = M_old;
        for (int s = 0; s < nsp; ++s) M = fmaxf(M, stage_p[(s * G_T + tid) * part_stride + rV]);
        const float f = (M_old == -INFINITY) ? 0.f : ex2(M_old - M);
        float lsum = (s0 == 0) ? 0.f : fin[G_T + tid] * f;
        for (int s = 0; s < nsp; ++s) {
          const float ms = stage_p[(s * G_T + tid) * part_stride + rV];
          if (ms != -INFINITY) lsum = fmaf(ex2(ms - M), stage_p[(s * G_T + tid) * part_stride + rV + 1], lsum);
        }
        fin[tid] = M;
        fin[G_T + tid] = lsum;
        fin[2 * G_T + tid] = f;  // rescale of what was accumulated before this chunk
      }
      __syncthreads();
      const bool final_chunk = s0 + nsp >= S;
      for (int idx = tid; idx < G_T * rV; idx += NT) {
        const int g = idx / rV, jj = idx - g * rV;
        const float M = fin[g];
        float o = (s0 == 0) ? 0.f : ot[idx] * fin[2 * G_T + g];
        if (M != -INFINITY)
          for (int s = 0; s < nsp; ++s) {
            const float ms = stage_p[(s * G_T + g) * part_stride + rV];
            if (ms != -INFINITY) o = fmaf(ex2(ms - M), stage_p[(s * G_T + g) * part_stride + jj], o);
          }
        if (final_chunk) {
          const float lsum = fin[G_T + g];
          o = lsum > 0.f ? o / lsum : 0.f;
        }
        ot[idx] = o;
      }
      __syncthreads();
    }
  }
  __syncthreads();

  // ---- up-projection o = o~ . P_V^T from shared memory, bf16 out --------------------------
  if (!mbar_wait_bounded(setup_bar, 1, a.dev_status)) return;
  {
    const uint32_t pv_addr = smem_u32(smem + L.region + L.pv);
    const int shv = (RV & 7) == 0 ? 0 : ((RV & 3) == 0 ? 1 : 2);
    for (int idx = tid; idx < gcount * d; idx += NT) {
      const int g = idx / d, i = idx - g * d;
      const uint32_t prow = pv_addr + (uint32_t)i * rV * 2u;
      const float* og = ot + g * rV;
      int c = ((i & 7) >> shv) % RV;
      float2 accv = f2(0.f, 0.f);
      for (int jj = 0; jj < RV; ++jj) {
        float2 pv[4];
        unpack8(lds128(prow + c * 16u), pv);
        const float4 x = *reinterpret_cast<const float4*>(og + c * 8);
        const float4 y = *reinterpret_cast<const float4*>(og + c * 8 + 4);
        accv = fma2(f2(x.x, x.y), pv[0], accv);
        accv = fma2(f2(x.z, x.w), pv[1], accv);
        accv = fma2(f2(y.x, y.y), pv[2], accv);
        accv = fma2(f2(y.z, y.w), pv[3], accv);
        c = (c + 1 == RV) ? 0 : c + 1;
      }
      a.out[((size_t)b * a.Hq + h0 + g) * d + i] = f32_to_bf16_rn(accv.x + accv.y);
    }
  }
}

// ------------------------------------------------------------------------------ launch

template <int G_T, int NP>
static cudaError_t launch_t(const DecodeArgs& a, cudaStream_t stream) {
  const DecodeSmem L = decode_smem_layout(NP, a.nstage, G_T, a.d, a.rK, a.rV);
  auto kern = stief_decode_kernel<G_T, NP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.S, a.Hkv * a.qsub, a.B);
  cfg.blockDim = dim3(NP * 64);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = a.pdl_first ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

uint32_t decode_smem_bytes(int NP, int nstage, int G_T, int d, int rK, int rV) {
  return decode_smem_layout(NP, nstage, G_T, d, rK, rV).total;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.G_T) {
    case 1: return a.npairs == 8 ? launch_t<1, 8>(a, stream) : launch_t<1, 4>(a, stream);
    case 2: return a.npairs == 8 ? launch_t<2, 8>(a, stream) : launch_t<2, 4>(a, stream);
    case 4: return a.npairs == 8 ? launch_t<4, 8>(a, stream) : launch_t<4, 4>(a, stream);
    case 8: return a.npairs == 8 ? launch_t<8, 8>(a, stream) : launch_t<8, 4>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace stief
