// compress_joint.cu -- append new tokens to a cache whose values are decomposed jointly over
// the KV heads (STAR-KV technical summary, "Metodologia" item 2, the hybrid decomposition):
// keys per head, k_lat[b][h][L + t] = bf16(k_new[b][h][t] . P_K[h]); values of all KV heads of
// a token together, v_joint[b][L + t] = bf16([v_new[b][0][t] | ... | v_new[b][Hkv-1][t]] . P_VJ).
//
//   stief_compress_joint_kernel -- the projections on CUDA cores.  grid (ceil(T/kJointRows),
//                                  Hkv + 1, B); blockIdx.y < Hkv projects that head's keys,
//                                  blockIdx.y == Hkv the joint value rows.  A thread owns one
//                                  output column for the block's rows; the input rows are
//                                  staged in shared memory (fp32) one chunk of the reduction
//                                  at a time, the basis is read row by row (coalesced over
//                                  the columns) from L2.
//   stief_joint_lens_kernel     -- the length update, launched after the projection in stream
//                                  order (every projection block has read the old lengths).
// Prefill-sized chunks (T >= 128) go to the tcgen05 projection instead
// (stief_compress_joint_tc_kernel, compress_joint_tc.cu) when its shared memory holds the
// whole joint basis, followed by the compress length kernel as a programmatic dependent.
//
// Every store is checked against the size of its tensor and skipped (reported as a capacity
// overflow) if it would fall outside; with valid lengths that never happens.
#include <cstdint>

#include "stief_device.cuh"
#include "stief_internal.h"

namespace stief {

constexpr int kJointRows = 8;       // new tokens per block
constexpr int kJointThreads = 128;  // one thread per output column (r <= 128)
constexpr int kJointChunk = 256;    // reduction elements staged per pass
constexpr int kJointTensorCoreMinRows = 128;  // T from which the tcgen05 path is used

__global__ void __launch_bounds__(kJointThreads) stief_compress_joint_kernel(const CompressArgs a) {
  __shared__ float xs[kJointRows][kJointChunk];
  const int b = blockIdx.z;
  const int z = blockIdx.y;  // KV head of the keys, or Hkv for the joint values
  const int t0 = blockIdx.x * kJointRows;
  const int L = __ldcg(a.seq_lens + b);
  // lengths outside [0, L_max - T] are reported by the length kernel; nothing is written here
  if (L < 0 || (long long)L + a.T > a.L_max) return;
  const int rows = min(kJointRows, a.T - t0);
  if (rows <= 0) return;
  const bool values = z == a.Hkv;
  const int ncols = values ? a.rV : a.rK;
  const int K_in = values ? a.Hkv * a.d : a.d;
  const uint16_t* P = values ? a.P_V : a.P_K + (size_t)z * a.d * a.rK;
  const int c = threadIdx.x;

  float acc[kJointRows];
#pragma unroll
  for (int t = 0; t < kJointRows; ++t) acc[t] = 0.f;

  for (int k0 = 0; k0 < K_in; k0 += kJointChunk) {
    const int kn = min(kJointChunk, K_in - k0);
    __syncthreads();  // the previous chunk has been consumed
    for (int i = threadIdx.x; i < kJointRows * kJointChunk; i += kJointThreads) {
      const int t = i / kJointChunk, k = i - t * kJointChunk;
      float x = 0.f;
      if (t < rows && k < kn) {
        const int j = k0 + k;  // input coordinate: head j / d, dimension j % d (values)
        const size_t src = values
            ? (((size_t)b * a.Hkv + j / a.d) * a.T + t0 + t) * a.d + (j % a.d)
            : (((size_t)b * a.Hkv + z) * a.T + t0 + t) * a.d + j;
        x = __uint_as_float((uint32_t)(values ? a.v_new : a.k_new)[src] << 16);
      }
      xs[t][k] = x;
    }
    __syncthreads();
    if (c < ncols) {
      for (int k = 0; k < kn; ++k) {
        const float p = __uint_as_float((uint32_t)__ldg(P + (size_t)(k0 + k) * ncols + c) << 16);
#pragma unroll
        for (int t = 0; t < kJointRows; ++t) acc[t] = fmaf(xs[t][k], p, acc[t]);
      }
    }
  }

  if (c >= ncols) return;
  const size_t total = values ? (size_t)a.B * a.L_max * a.rV
                              : (size_t)a.B * a.Hkv * a.L_max * a.rK;
  uint16_t* out = values ? a.v_lat : a.k_lat;
#pragma unroll
  for (int t = 0; t < kJointRows; ++t) {
    if (t >= rows) break;
    const size_t row = values ? (size_t)b * a.L_max + L + t0 + t
                              : ((size_t)b * a.Hkv + z) * a.L_max + L + t0 + t;
    const size_t dst = row * ncols + c;
    if (dst < total) out[dst] = f32_to_bf16_rn(acc[t]);
    else report(a.dev_status, STIEF_DEV_CAPACITY_OVERFLOW);
  }
}

__global__ void __launch_bounds__(256) stief_joint_lens_kernel(const CompressArgs a) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= a.B) return;
  const int L = a.seq_lens[b];
  if (L < 0) report(a.dev_status, STIEF_DEV_BAD_LENGTH);
  else if ((long long)L + a.T > a.L_max) report(a.dev_status, STIEF_DEV_CAPACITY_OVERFLOW);
  else a.seq_lens[b] = L + a.T;
}

cudaError_t launch_compress_joint(const CompressArgs& a, cudaStream_t stream) {
  if (a.T >= kJointTensorCoreMinRows && compress_joint_tc_fits(a.Hkv, a.rK, a.rV)) {
    cudaError_t e = launch_compress_joint_tc(a, stream);
    if (e == cudaSuccess) e = launch_seq_lens(a, stream);
    // the length kernel lets its dependents start early: a decode that follows must not
    // request cache tiles before its dependency wait
    if (e == cudaSuccess) mark_stream_compress(a.device, stream, true);
    return e;
  }
  const dim3 grid((a.T + kJointRows - 1) / kJointRows, a.Hkv + 1, a.B);
  stief_compress_joint_kernel<<<grid, kJointThreads, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  stief_joint_lens_kernel<<<(a.B + 255) / 256, 256, 0, stream>>>(a);
  e = cudaGetLastError();
  // these kernels let no dependent start early: a decode that follows may read ahead
  if (e == cudaSuccess) mark_stream_compress(a.device, stream, false);
  return e;
}

}  // namespace stief
