// compress_kernels.cu -- compressed storage of new key/value rows, for sm_100a.
//
// Operation (StiefAttention technical summary, "Mecanismo Central" item 5):
// keys and values are stored compressed, K_down = K P_K and V_down = V P_V.
// For every (sequence b, KV head h) the T new rows are projected with fp32
// accumulation, rounded once to bf16 (RNE) and written at rows
// [seq_lens[b], seq_lens[b] + T) of the latent cache; then seq_lens[b] += T.
//
// Kernels:
//   stief_compress_rows_kernel  -- CUDA-core projection, grid (ceil(T/TT), 2 Hkv, B);
//                                  used for decode-sized appends (small T)
//   stief_compress_tc_kernel    -- tcgen05 tensor-core projection of prefill-sized
//                                  chunks (T >= 128), compress_tc.cu
//   stief_seq_lens_kernel       -- the length update, launched as a programmatic
//                                  dependent of the projection so that it runs
//                                  only after every projection CTA has read the
//                                  old lengths
#include <cstdint>

#include "stief_device.cuh"
#include "stief_internal.h"

namespace stief {

constexpr int kRowsPerCta = 8;  // new rows per CTA of the CUDA-core path (T > 1)
constexpr int kTensorCoreMinRows = 128;  // T from which the tcgen05 path is used
constexpr int kSmallThreads = 256;

__device__ __forceinline__ float2 fma2c(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// CUDA-core projection of up to TT new rows of one (sequence, KV head, K or V).
// grid (ceil(T/TT), Hkv * 2, B); blockIdx.y = 2 * head + (0: keys, 1: values).
// The basis and the rows arrive by bulk copy; thread = (column pair, slice of d);
// slices are summed through shared memory.
template <int TT>
__global__ void __launch_bounds__(kSmallThreads) stief_compress_rows_kernel(const CompressArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x;
  const int h = blockIdx.y >> 1;
  const bool is_v = blockIdx.y & 1;
  const int b = blockIdx.z;
  const int d = a.d, T = a.T;
  const int r = is_v ? a.rV : a.rK;
  const int r0 = blockIdx.x * TT;
  const int nrows = min(TT, T - r0);
  const uint16_t* P = (is_v ? a.P_V : a.P_K) + (size_t)h * d * r;
  const uint16_t* X = (is_v ? a.v_new : a.k_new) + (((size_t)b * a.Hkv + h) * T + r0) * d;

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  uint16_t* ps = reinterpret_cast<uint16_t*>(smem + 128);
  uint16_t* xs = ps + d * r;
  float2* red = reinterpret_cast<float2*>(xs + TT * d);

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
    const uint32_t pb = 2u * d * r, xb = 2u * nrows * d;
    mbar_arrive_expect_tx(bar, pb + xb);
    bulk_g2s(ps, P, pb, bar);
    bulk_g2s(xs, X, xb, bar);
  }
  pdl_launch_dependents();

  const int Lb = a.seq_lens[b];
  const bool bad = Lb < 0 || Lb > a.L_max;
  const CacheRows cr{a.block_table, a.max_pages, a.page_size, a.num_pages, a.Hkv, a.L_max};
  // no room, or (paged) a page of the new rows is not mapped: the sequence is not appended to
  const bool full = !bad && ((long long)Lb + T > a.L_max || !pages_mapped(cr, b, Lb, Lb + T));
  if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0) {
    if (bad) report(a.dev_status, STIEF_DEV_BAD_LENGTH);
    if (full) report(a.dev_status, STIEF_DEV_CAPACITY_OVERFLOW);
  }
  __syncthreads();  // barrier initialised before anyone waits on it
  const bool ok = mbar_wait_bounded(bar, 0, a.dev_status);
  if (bad || full || !ok) return;  // the copies have landed (or the wait gave up)

  const int pairs = r / 2;  // 8 .. 64
  int slices = 1;           // a power of two with pairs * slices <= 256 (so it divides d)
  while (pairs * slices * 2 <= kSmallThreads) slices *= 2;
  const int rows_per_slice = d / slices;
  const int cp = tid % pairs, sl = tid / pairs;
  const bool active = sl < slices;
  const uint32_t* P2 = reinterpret_cast<const uint32_t*>(ps);
  float2 acc[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = make_float2(0.f, 0.f);
  for (int i = sl * rows_per_slice; active && i < (sl + 1) * rows_per_slice; ++i) {
    const uint32_t pw = P2[i * pairs + cp];
    const float2 pf = make_float2(bf16lo(pw), bf16hi(pw));
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      const float xv = bf16_to_f32(xs[t * d + i]);
      acc[t] = fma2c(make_float2(xv, xv), pf, acc[t]);
    }
  }
  if (active) {
#pragma unroll
    for (int t = 0; t < TT; ++t) red[(sl * TT + t) * pairs + cp] = acc[t];
  }
  __syncthreads();
  uint32_t* lat = reinterpret_cast<uint32_t*>(is_v ? a.v_lat : a.k_lat);
  const bool q8 = a.k_scale != nullptr;
  for (int o = tid; o < nrows * pairs; o += kSmallThreads) {
    const int t = o / pairs, c2 = o - t * pairs;
    float2 sum = make_float2(0.f, 0.f);
    for (int s2 = 0; s2 < slices; ++s2) {
      const float2 v = red[(s2 * TT + t) * pairs + c2];
      sum.x += v.x;
      sum.y += v.y;
    }
    if (q8)  // keep the bf16-rounded row for the quantisation below (slice 0's own slot)
      red[t * pairs + c2] = make_float2(bf16_round(sum.x), bf16_round(sum.y));
    else
      lat[cache_row(cr, b, h, Lb + r0 + t) * pairs + c2] = pack_bf16x2_rn(sum.x, sum.y);
  }
  if (q8) {
    // int8 / 4-bit cache: a thread per row: one fp32 scale (max / 127, or max / 7) and RNE
    // codes; 4-bit codes two per byte, column 2 j in the low nibble of byte j
    __syncthreads();
    if (tid < nrows) {
      const float* row = reinterpret_cast<const float*>(red + tid * pairs);
      const int qmax = a.q4 ? 7 : 127;
      float amax = 0.f;
      for (int c = 0; c < r; ++c) amax = fmaxf(amax, fabsf(row[c]));
      const float scale = __fdiv_rn(amax, (float)qmax);
      const long long crow = cache_row(cr, b, h, Lb + r0 + tid);
      if (a.q4) {
        uint8_t* dst = reinterpret_cast<uint8_t*>(is_v ? a.v_lat : a.k_lat) + crow * (r / 2);
        for (int c = 0; c < r; c += 2)
          dst[c / 2] = (uint8_t)((quantize_code(row[c], scale, 7) & 0xF) |
                                 ((quantize_code(row[c + 1], scale, 7) & 0xF) << 4));
      } else {
        int8_t* dst = reinterpret_cast<int8_t*>(is_v ? a.v_lat : a.k_lat) + crow * r;
        for (int c = 0; c < r; ++c) dst[c] = (int8_t)quantize_code(row[c], scale);
      }
      (is_v ? a.v_scale : a.k_scale)[crow] = scale;
    }
  }
}

__global__ void __launch_bounds__(256) stief_seq_lens_kernel(const CompressArgs a) {
  // the next kernel may start now: its inputs are read only after its own dependency wait
  // (which waits for this grid, and so for the projection), and a decode launched right after
  // a compress reads no cache tile before that wait (the library marks the stream)
  pdl_launch_dependents();
  pdl_wait();  // every projection CTA has finished reading the old lengths
  const CacheRows cr{a.block_table, a.max_pages, a.page_size, a.num_pages, a.Hkv, a.L_max};
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < a.B; b += gridDim.x * blockDim.x) {
    const int L = a.seq_lens[b];
    if (L >= 0 && (long long)L + a.T <= a.L_max && pages_mapped(cr, b, L, L + a.T))
      a.seq_lens[b] = L + a.T;
  }
}

cudaError_t launch_seq_lens(const CompressArgs& a, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.B + 255) / 256);
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, stief_seq_lens_kernel, a);
}

template <int TT>
static cudaError_t launch_rows(const CompressArgs& a, cudaStream_t stream) {
  const int rmax = a.rK > a.rV ? a.rK : a.rV;
  const uint32_t smem = 128u + 2u * a.d * rmax + 2u * TT * a.d + 8u * TT * kSmallThreads;
  static SmemLimit limit;
  cudaError_t e = limit.ensure(reinterpret_cast<const void*>(stief_compress_rows_kernel<TT>),
                               a.device, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.T + TT - 1) / TT, a.Hkv * 2, a.B);
  stief_compress_rows_kernel<TT><<<grid, kSmallThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_compress_tc(const CompressArgs& a, cudaStream_t stream);

cudaError_t launch_compress(const CompressArgs& a, cudaStream_t stream) {
  cudaError_t e;
  if (a.T >= kTensorCoreMinRows)
    e = launch_compress_tc(a, stream);
  else
    e = (a.T == 1) ? launch_rows<1>(a, stream) : launch_rows<kRowsPerCta>(a, stream);
  if (e != cudaSuccess) return e;
  e = launch_seq_lens(a, stream);
  if (e == cudaSuccess) mark_stream_compress(a.device, stream, true);
  return e;
}

}  // namespace stief
