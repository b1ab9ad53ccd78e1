// decode_kernels.cu -- split-KV decode attention over the latent (Stiefel-projected)
// KV cache, for sm_100a.
//
// Operation (StiefAttention technical summary, "Mecanismo Central" item 5): keys
// and values are stored as K_down = K P_K, V_down = V P_V and attention runs over
// the reconstructions K~ = K_down P_K^T, V~ = V_down P_V^T.  The kernels never
// form K~ or V~; they use the equal products
//     s_t = (q P_K) . K_down[t] / sqrt(d)          (query projected once per CTA)
//     o   = (sum_t softmax(s)_t V_down[t]) P_V^T   (up-projection after the mix)
// so the HBM stream is the bf16 latent cache, read once per KV head.
//
// Kernel 1 (stief_decode_split_kernel), grid (splits, Hkv * qsub, B):
//   one CTA serves up to G_T query heads of one KV head over one token range.
//   - q~ = q . P_K * log2(e)/sqrt(d) in fp32 (shared memory, padded chunk-major)
//   - every warp streams its own 32-token tiles of K_down and V_down through a
//     private ring of shared-memory stages filled by 1-D bulk copies (TMA engine)
//     that complete on per-stage mbarriers; no CTA-wide barrier in the loop
//   - scores: one lane per token; each lane walks the 16-byte chunks of its row
//     in a lane-rotated order so the 8 lanes of a shared-memory phase hit 8
//     different bank groups, while q~ is read with broadcasts
//   - online softmax in the log2 domain with lazy rescaling: accumulators are
//     rescaled only when a score exceeds the running reference by more than 8
//     (so every weight stays <= 2^8 in fp32)
//   - latent value mix: r_V/8 lanes per token, 8 values per lane, fp32 FMA
//   - partial (m, l, o~[r_V]) per (query head, split) written to the workspace
// Kernel 2 (stief_decode_combine_kernel), grid (Hkv * qsub, B), launched as a
// programmatic dependent: log-sum-exp merge of the splits, division by the sum,
// up-projection o~ . P_V^T, bf16 store.
#include <cfloat>
#include <cmath>
#include <cstdint>

#include "stief_device.cuh"
#include "stief_internal.h"

namespace stief {

constexpr int kTile = 32;            // tokens per warp tile
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

// Shared-memory carve-up of the split kernel (byte offsets from the dynamic base).
struct SplitSmem {
  uint32_t bars;    // (NW * nstage + 1) mbarriers
  uint32_t q;       // G_T x d bf16 query rows
  uint32_t pk;      // d x rK bf16 basis
  uint32_t qt;      // (rK/8) chunks x (G_T*8 + 4) fp32 projected, scaled queries
  uint32_t p;       // NW x 32 x G_T fp32 softmax weights of the current tile
  uint32_t ml;      // NW x G_T x 2 fp32 per-warp (m, l)
  uint32_t region;  // stage buffers, reused for the cross-warp reduction
  uint32_t total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline SplitSmem split_smem_layout(int NW, int nstage, int G_T, int d, int rK,
                                                       int rV) {
  SplitSmem s;
  uint32_t off = 0;
  s.bars = off;
  off = align_up(off + 8u * (NW * nstage + 1), 128);
  s.q = off;
  off = align_up(off + 2u * G_T * d, 128);
  s.pk = off;
  off = align_up(off + 2u * d * rK, 128);
  s.qt = off;
  off = align_up(off + 4u * (rK / 8) * (G_T * 8 + 4), 128);
  s.p = off;
  off = align_up(off + 4u * NW * kTile * G_T, 128);
  s.ml = off;
  off = align_up(off + 8u * NW * G_T, 128);
  s.region = off;
  const uint32_t stage = (uint32_t)NW * nstage * kTile * (rK + rV) * 2u;
  const uint32_t red = (uint32_t)NW * 32u * G_T * 8u * 4u;
  off = align_up(off + (stage > red ? stage : red), 128);
  s.total = off;
  return s;
}

template <int G_T, int NW>
__global__ void __launch_bounds__(NW * 32, 1) stief_decode_split_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int s_idx = blockIdx.x;                 // split
  const int kvh = blockIdx.y / a.qsub;          // KV head
  const int qs = blockIdx.y - kvh * a.qsub;     // query sub-group of that head
  const int b = blockIdx.z;
  const int d = a.d, rK = a.rK, rV = a.rV, S = a.S;
  const int nstage = a.nstage;
  const int h0 = kvh * a.G + qs * G_T;          // first query head of this CTA
  const int gcount = min(G_T, a.G - qs * G_T);  // valid query heads here

  const SplitSmem L = split_smem_layout(NW, nstage, G_T, d, rK, rV);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* setup_bar = bars + NW * nstage;
  const uint32_t tile_bytes = (uint32_t)kTile * (rK + rV) * 2u;
  uint8_t* my_stages = smem + L.region + (size_t)warp * nstage * tile_bytes;

  if (tid == 0) {
    for (int i = 0; i < NW * nstage + 1; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
  __syncthreads();

  // Query rows and the key basis: independent of any earlier kernel in this call.
  if (tid == 0) {
    const uint32_t qbytes = 2u * gcount * d;
    const uint32_t pbytes = 2u * d * rK;
    mbar_arrive_expect_tx(setup_bar, qbytes + pbytes);
    bulk_g2s(smem + L.q, a.q + ((size_t)b * a.Hq + h0) * d, qbytes, setup_bar);
    bulk_g2s(smem + L.pk, a.P_K + (size_t)kvh * d * rK, pbytes, setup_bar);
  }
  pdl_launch_dependents();

  // Everything below may read what the preceding kernel in the stream wrote.
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
  const int my_tiles = warp < n_tiles ? (n_tiles - warp + NW - 1) / NW : 0;

  const size_t head_row0 = ((size_t)b * a.Hkv + kvh) * a.L_max;
  const uint16_t* kbase_g = a.k_lat + head_row0 * rK;
  const uint16_t* vbase_g = a.v_lat + head_row0 * rV;
  const uint64_t policy = l2_policy_evict_first();

  auto issue = [&](int k) {  // tile k of this warp into stage k % nstage (lane 0 only)
    const int j = warp + k * NW;
    const int tok0 = t0 + j * kTile;
    const int n = min(kTile, t1 - tok0);
    uint8_t* st = my_stages + (size_t)(k % nstage) * tile_bytes;
    uint64_t* bar = &bars[warp * nstage + (k % nstage)];
    const uint32_t kb = (uint32_t)n * rK * 2u, vb = (uint32_t)n * rV * 2u;
    mbar_arrive_expect_tx(bar, kb + vb);
    bulk_g2s_hint(st, kbase_g + (size_t)tok0 * rK, kb, bar, policy);
    bulk_g2s_hint(st + (size_t)kTile * rK * 2, vbase_g + (size_t)tok0 * rV, vb, bar, policy);
  };
  if (lane == 0) {
    const int pre = min(nstage, my_tiles);
    for (int k = 0; k < pre; ++k) issue(k);
  }

  // ---- q~ = q . P_K, scaled into the log2 domain ---------------------------------
  bool ok = mbar_wait_bounded(setup_bar, 0, a.dev_status);
  const float qscale = a.qscale;
  {
    const int RK = rK / 8;
    const int qstride = G_T * 8 + 4;  // floats per chunk row (odd multiple of 16 bytes)
    const uint16_t* qs_ = reinterpret_cast<const uint16_t*>(smem + L.q);
    const uint16_t* pk = reinterpret_cast<const uint16_t*>(smem + L.pk);
    float* qt = reinterpret_cast<float*>(smem + L.qt);
    for (int idx = tid; idx < G_T * rK; idx += NW * 32) {
      const int g = idx / rK, c = idx - g * rK;
      float acc = 0.f;
      if (ok && g < gcount) {
        const uint16_t* qrow = qs_ + g * d;
#pragma unroll 8
        for (int i = 0; i < d; ++i) acc = fmaf(bf16_to_f32(qrow[i]), bf16_to_f32(pk[i * rK + c]), acc);
      }
      qt[(c >> 3) * qstride + g * 8 + (c & 7)] = acc * qscale;
    }
    (void)RK;
  }
  __syncthreads();

  // ---- streaming loop (per warp) ----------------------------------------------------
  const int RK = rK >> 3;
  const int RV = rV >> 3;
  const int sh = (RK & 7) == 0 ? 0 : ((RK & 3) == 0 ? 1 : 2);
  const int delta = (lane & 7) >> sh;
  const uint32_t qstride_b = (uint32_t)(G_T * 8 + 4) * 4u;
  const uint32_t qt_addr = smem_u32(smem + L.qt);
  float* p_tile = reinterpret_cast<float*>(smem + L.p) + warp * kTile * G_T;
  const uint32_t p_addr = smem_u32(p_tile);
  const int TPW = 32 / RV;            // tokens per value step
  const int vslot = lane / RV;
  const int vchunk = lane - vslot * RV;
  const bool vactive = vslot < TPW;

  float m_ref[G_T], l_lane[G_T], acc[G_T][8];
#pragma unroll
  for (int g = 0; g < G_T; ++g) {
    m_ref[g] = -INFINITY;
    l_lane[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
  }

  int k_done = 0;
  for (int k = 0; k < my_tiles && ok; ++k) {
    const int stg = k % nstage;
    if (!mbar_wait_bounded(&bars[warp * nstage + stg], (uint32_t)((k / nstage) & 1), a.dev_status)) {
      ok = false;
      break;
    }
    k_done = k + 1;
    const int tok0 = t0 + (warp + k * NW) * kTile;
    const int n = min(kTile, t1 - tok0);
    uint8_t* st = my_stages + (size_t)stg * tile_bytes;
    const uint32_t kst = smem_u32(st);
    const uint32_t vst = kst + (uint32_t)kTile * rK * 2u;

    // scores: lane = token
    float s[G_T];
#pragma unroll
    for (int g = 0; g < G_T; ++g) s[g] = 0.f;
    {
      const uint32_t krow = kst + (uint32_t)lane * rK * 2u;
      int c = delta;
      for (int jj = 0; jj < RK; ++jj) {
        const uint4 kv = lds128(krow + c * 16u);
        const float k0 = bf16lo(kv.x), k1 = bf16hi(kv.x), k2 = bf16lo(kv.y), k3 = bf16hi(kv.y);
        const float k4 = bf16lo(kv.z), k5 = bf16hi(kv.z), k6 = bf16lo(kv.w), k7 = bf16hi(kv.w);
        const uint32_t qa = qt_addr + (uint32_t)c * qstride_b;
#pragma unroll
        for (int g = 0; g < G_T; ++g) {
          const float4 x = lds128f(qa + g * 32u);
          const float4 y = lds128f(qa + g * 32u + 16u);
          float t = s[g];
          t = fmaf(x.x, k0, t);
          t = fmaf(x.y, k1, t);
          t = fmaf(x.z, k2, t);
          t = fmaf(x.w, k3, t);
          t = fmaf(y.x, k4, t);
          t = fmaf(y.y, k5, t);
          t = fmaf(y.z, k6, t);
          t = fmaf(y.w, k7, t);
          s[g] = t;
        }
        c = (c + 1 == RK) ? 0 : c + 1;
      }
    }
    // online softmax (log2 domain), lazy rescale
    const bool valid = lane < n;
    float pw_own[G_T];
#pragma unroll
    for (int g = 0; g < G_T; ++g) {
      const float sg = valid ? s[g] : -INFINITY;
      if (__any_sync(0xffffffffu, sg > m_ref[g] + kRescaleTau)) {
        const float m_new = fmaxf(m_ref[g], warp_max(sg));
        const float f = ex2(m_ref[g] - m_new);  // 0 when m_ref was -inf
        l_lane[g] *= f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] *= f;
        m_ref[g] = m_new;
      }
      pw_own[g] = valid ? ex2(sg - m_ref[g]) : 0.f;
      l_lane[g] += pw_own[g];
    }
    if constexpr (G_T >= 4) {
#pragma unroll
      for (int g4 = 0; g4 < G_T; g4 += 4)
        *reinterpret_cast<float4*>(p_tile + lane * G_T + g4) =
            make_float4(pw_own[g4], pw_own[g4 + 1], pw_own[g4 + 2], pw_own[g4 + 3]);
    } else {
#pragma unroll
      for (int g = 0; g < G_T; ++g) p_tile[lane * G_T + g] = pw_own[g];
    }
    __syncwarp();

    // latent value mix: RV lanes per token
    if (vactive) {
      for (int t = vslot; t < n; t += TPW) {
        const uint4 vv = lds128(vst + (uint32_t)t * rV * 2u + vchunk * 16u);
        float v[8] = {bf16lo(vv.x), bf16hi(vv.x), bf16lo(vv.y), bf16hi(vv.y),
                      bf16lo(vv.z), bf16hi(vv.z), bf16lo(vv.w), bf16hi(vv.w)};
        float pw[G_T];
        if constexpr (G_T >= 4) {
#pragma unroll
          for (int g4 = 0; g4 < G_T; g4 += 4) {
            const float4 pp = lds128f(p_addr + (uint32_t)(t * G_T + g4) * 4u);
            pw[g4] = pp.x;
            pw[g4 + 1] = pp.y;
            pw[g4 + 2] = pp.z;
            pw[g4 + 3] = pp.w;
          }
        } else {
#pragma unroll
          for (int g = 0; g < G_T; ++g) pw[g] = p_tile[t * G_T + g];
        }
#pragma unroll
        for (int g = 0; g < G_T; ++g)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pw[g], v[e], acc[g][e]);
      }
    }
    __syncwarp();
    if (lane == 0 && k + nstage < my_tiles) issue(k + nstage);
  }

  // After a timed-out wait: give the copies still in flight a bounded chance to land
  // before this CTA's shared memory is released.
  if (!ok && lane == 0) {
    for (int k = k_done; k < min(my_tiles, k_done + nstage); ++k)
      mbar_wait_bounded(&bars[warp * nstage + (k % nstage)], (uint32_t)((k / nstage) & 1), nullptr);
    if (warp == 0) mbar_wait_bounded(setup_bar, 0, nullptr);
  }

  // ---- cross-warp merge --------------------------------------------------------------
  float* ml = reinterpret_cast<float*>(smem + L.ml);
#pragma unroll
  for (int g = 0; g < G_T; ++g) {
    const float lw = warp_sum(l_lane[g]);
    if (lane == 0) {
      ml[(warp * G_T + g) * 2 + 0] = m_ref[g];
      ml[(warp * G_T + g) * 2 + 1] = lw;
    }
  }
  __syncthreads();  // every warp is done with its stages: the region becomes the reduction buffer
  float* red = reinterpret_cast<float*>(smem + L.region);
  {
    float* mine = red + ((size_t)warp * 32 + lane) * G_T * 8;
#pragma unroll
    for (int g = 0; g < G_T; ++g)
#pragma unroll
      for (int e = 0; e < 8; ++e) mine[g * 8 + e] = vactive ? acc[g][e] : 0.f;
  }
  __syncthreads();

  const size_t unit = ((size_t)b * a.Hkv + kvh) * a.qsub + qs;
  for (int idx = tid; idx < G_T * rV; idx += NW * 32) {
    const int g = idx / rV, jj = idx - g * rV;
    const int c = jj >> 3, e = jj & 7;
    float M = -INFINITY;
    for (int w = 0; w < NW; ++w) M = fmaxf(M, ml[(w * G_T + g) * 2]);
    float o = 0.f, lsum = 0.f;
    for (int w = 0; w < NW; ++w) {
      const float mw = ml[(w * G_T + g) * 2];
      const float sc = (mw == -INFINITY) ? 0.f : ex2(mw - M);
      float part = 0.f;
      for (int slot = 0; slot < TPW; ++slot)
        part += red[((size_t)w * 32 + slot * RV + c) * G_T * 8 + g * 8 + e];
      o = fmaf(sc, part, o);
      lsum = fmaf(sc, ml[(w * G_T + g) * 2 + 1], lsum);
    }
    const size_t pi = (unit * S + s_idx) * G_T + g;
    a.ws_o[pi * rV + jj] = o;
    if (jj == 0) {
      a.ws_ml[pi * 2 + 0] = M;
      a.ws_ml[pi * 2 + 1] = lsum;
    }
  }
}

// Combine the splits and up-project: out[b][h] = bf16( (sum_s w_s o~_s / sum_s w_s l_s) . P_V^T ).
template <int G_T>
__global__ void __launch_bounds__(128) stief_decode_combine_kernel(const DecodeArgs a) {
  __shared__ float ot[G_T][128];
  const int tid = threadIdx.x;
  const int kvh = blockIdx.x / a.qsub;
  const int qs = blockIdx.x - kvh * a.qsub;
  const int b = blockIdx.y;
  const int rV = a.rV, S = a.S, d = a.d;
  const int h0 = kvh * a.G + qs * G_T;
  const int gcount = min(G_T, a.G - qs * G_T);
  const size_t unit = ((size_t)b * a.Hkv + kvh) * a.qsub + qs;

  pdl_wait();

  for (int idx = tid; idx < gcount * rV; idx += blockDim.x) {
    const int g = idx / rV, jj = idx - g * rV;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, a.ws_ml[((unit * S + s) * G_T + g) * 2]);
    float o = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
      for (int s = 0; s < S; ++s) {
        const size_t pi = (unit * S + s) * G_T + g;
        const float ms = a.ws_ml[pi * 2];
        if (ms == -INFINITY) continue;
        const float w = ex2(ms - M);
        lsum = fmaf(w, a.ws_ml[pi * 2 + 1], lsum);
        o = fmaf(w, a.ws_o[pi * rV + jj], o);
      }
    }
    ot[g][jj] = lsum > 0.f ? o / lsum : 0.f;
  }
  __syncthreads();

  for (int i = tid; i < d; i += blockDim.x) {
    const uint4* prow = reinterpret_cast<const uint4*>(a.P_V + ((size_t)kvh * d + i) * rV);
    float accs[G_T];
#pragma unroll
    for (int g = 0; g < G_T; ++g) accs[g] = 0.f;
    for (int c = 0; c < rV / 8; ++c) {
      const uint4 pv = prow[c];
      const float p8[8] = {bf16lo(pv.x), bf16hi(pv.x), bf16lo(pv.y), bf16hi(pv.y),
                           bf16lo(pv.z), bf16hi(pv.z), bf16lo(pv.w), bf16hi(pv.w)};
#pragma unroll
      for (int g = 0; g < G_T; ++g)
#pragma unroll
        for (int e = 0; e < 8; ++e) accs[g] = fmaf(ot[g][c * 8 + e], p8[e], accs[g]);
    }
    for (int g = 0; g < gcount; ++g)
      a.out[((size_t)b * a.Hq + h0 + g) * d + i] = f32_to_bf16_rn(accs[g]);
  }
}

// ------------------------------------------------------------------------------ launch

template <int G_T, int NW>
static cudaError_t launch_split(const DecodeArgs& a, cudaStream_t stream, bool pdl) {
  const SplitSmem L = split_smem_layout(NW, a.nstage, G_T, a.d, a.rK, a.rV);
  auto kern = stief_decode_split_kernel<G_T, NW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.S, a.Hkv * a.qsub, a.B);
  cfg.blockDim = dim3(NW * 32);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int G_T>
static cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.Hkv * a.qsub, a.B);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, stief_decode_combine_kernel<G_T>, a);
}

uint32_t decode_split_smem_bytes(int NW, int nstage, int G_T, int d, int rK, int rV) {
  return split_smem_layout(NW, nstage, G_T, d, rK, rV).total;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  cudaError_t e;
#define STIEF_SPLIT(GT)                                                        \
  case GT:                                                                     \
    e = (a.nwarps == 8) ? launch_split<GT, 8>(a, stream, a.pdl_first)          \
                        : launch_split<GT, 4>(a, stream, a.pdl_first);         \
    if (e != cudaSuccess) return e;                                            \
    return launch_combine<GT>(a, stream);
  switch (a.G_T) {
    STIEF_SPLIT(1)
    STIEF_SPLIT(2)
    STIEF_SPLIT(4)
    STIEF_SPLIT(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef STIEF_SPLIT
}

}  // namespace stief
