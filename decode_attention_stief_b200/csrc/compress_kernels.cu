// compress_kernels.cu -- compressed storage of new key/value rows, for sm_100a.
//
// Operation (StiefAttention technical summary, "Mecanismo Central" item 5):
// keys and values are stored compressed, K_down = K P_K and V_down = V P_V.
// For every (sequence b, KV head h) the T new rows are projected with fp32
// accumulation, rounded once to bf16 (RNE) and written at rows
// [seq_lens[b], seq_lens[b] + T) of the latent cache; then seq_lens[b] += T.
//
// Kernels:
//   stief_compress_rows_kernel  -- CUDA-core projection, grid (ceil(T/TT), Hkv, B);
//                                  used for decode-sized appends (small T)
//   stief_seq_lens_kernel       -- the length update, launched as a programmatic
//                                  dependent of the projection so that it runs
//                                  only after every projection CTA has read the
//                                  old lengths
#include <cstdint>

#include "stief_device.cuh"
#include "stief_internal.h"

namespace stief {

constexpr int kRowsPerCta = 8;  // TT: new rows handled by one CTA of the CUDA-core path

// Shared memory: P_K[h] (d x rK), P_V[h] (d x rV), then TT rows of k and of v.
__global__ void __launch_bounds__(256) stief_compress_rows_kernel(const CompressArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int d = a.d, rK = a.rK, rV = a.rV, T = a.T;
  const int r0 = blockIdx.x * kRowsPerCta;
  const int nrows = min(kRowsPerCta, T - r0);

  pdl_launch_dependents();

  const int Lb = a.seq_lens[b];
  if (Lb < 0 || Lb > a.L_max) {
    if (tid == 0 && blockIdx.x == 0 && h == 0) report(a.dev_status, STIEF_DEV_BAD_LENGTH);
    return;
  }
  if ((long long)Lb + T > a.L_max) {
    if (tid == 0 && blockIdx.x == 0 && h == 0) report(a.dev_status, STIEF_DEV_CAPACITY_OVERFLOW);
    return;
  }

  uint16_t* pk = reinterpret_cast<uint16_t*>(smem);
  uint16_t* pv = pk + d * rK;
  uint16_t* xk = pv + d * rV;
  uint16_t* xv = xk + kRowsPerCta * d;
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.P_K + (size_t)h * d * rK);
    uint4* dst = reinterpret_cast<uint4*>(pk);
    for (int i = tid; i < d * rK / 8; i += blockDim.x) dst[i] = src[i];
    src = reinterpret_cast<const uint4*>(a.P_V + (size_t)h * d * rV);
    dst = reinterpret_cast<uint4*>(pv);
    for (int i = tid; i < d * rV / 8; i += blockDim.x) dst[i] = src[i];
    const size_t row0 = (((size_t)b * a.Hkv + h) * T + r0) * d;
    src = reinterpret_cast<const uint4*>(a.k_new + row0);
    dst = reinterpret_cast<uint4*>(xk);
    for (int i = tid; i < nrows * d / 8; i += blockDim.x) dst[i] = src[i];
    src = reinterpret_cast<const uint4*>(a.v_new + row0);
    dst = reinterpret_cast<uint4*>(xv);
    for (int i = tid; i < nrows * d / 8; i += blockDim.x) dst[i] = src[i];
  }
  __syncthreads();

  // threads [0, 128): key column tid; threads [128, 256): value column tid - 128
  const bool is_v = tid >= 128;
  const int c = is_v ? tid - 128 : tid;
  const int r = is_v ? rV : rK;
  if (c >= r) return;
  const uint16_t* P = is_v ? pv : pk;
  const uint16_t* X = is_v ? xv : xk;
  float acc[kRowsPerCta];
#pragma unroll
  for (int t = 0; t < kRowsPerCta; ++t) acc[t] = 0.f;
  for (int i = 0; i < d; ++i) {
    const float p = bf16_to_f32(P[i * r + c]);
#pragma unroll
    for (int t = 0; t < kRowsPerCta; ++t) acc[t] = fmaf(bf16_to_f32(X[t * d + i]), p, acc[t]);
  }
  uint16_t* dst = (is_v ? a.v_lat : a.k_lat) + (((size_t)b * a.Hkv + h) * a.L_max + Lb + r0) * r;
  for (int t = 0; t < nrows; ++t) dst[(size_t)t * r + c] = f32_to_bf16_rn(acc[t]);
}

__global__ void __launch_bounds__(256) stief_seq_lens_kernel(int32_t* seq_lens, int B, int T,
                                                             int L_max) {
  pdl_wait();  // every projection CTA has finished reading the old lengths
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x) {
    const int L = seq_lens[b];
    if (L >= 0 && (long long)L + T <= L_max) seq_lens[b] = L + T;
  }
}

static cudaError_t launch_seq_lens(const CompressArgs& a, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.B + 255) / 256);
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, stief_seq_lens_kernel, a.seq_lens, a.B, a.T, a.L_max);
}

cudaError_t launch_compress(const CompressArgs& a, cudaStream_t stream) {
  const uint32_t smem = 2u * (a.d * (a.rK + a.rV) + 2 * kRowsPerCta * a.d);
  cudaError_t e = cudaFuncSetAttribute(stief_compress_rows_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.T + kRowsPerCta - 1) / kRowsPerCta, a.Hkv, a.B);
  stief_compress_rows_kernel<<<grid, 256, smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_seq_lens(a, stream);
}

}  // namespace stief
