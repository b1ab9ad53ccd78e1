// stief_internal.h -- argument blocks and launch entry points shared between the
// C-ABI host code (stief_api.cu) and the kernel files.  Not a public header.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace stief {

// Everything the decode kernels need, validated by the host code.
struct DecodeArgs {
  const uint16_t* q;
  const uint16_t* P_K;
  const uint16_t* P_V;
  const uint16_t* k_lat;
  const uint16_t* v_lat;
  const int32_t* seq_lens;
  uint16_t* out;
  float* ws_o;   // [units * S * G_T][rV] unnormalised partial latent outputs
  float* ws_ml;  // [units * S * G_T][2]  partial (running max, sum), log2 domain
  uint32_t* dev_status;
  int B, Hq, Hkv, G, G_T, qsub, d, rK, rV, L_max, S;
  int nwarps;     // warps per split CTA (4 or 8)
  int nstage;     // shared-memory stages per warp
  float qscale;   // log2(e) / sqrt(d), applied to q . P_K
  bool pdl_first; // launch the split kernel as a programmatic dependent
};

struct CompressArgs {
  const uint16_t* k_new;
  const uint16_t* v_new;
  const uint16_t* P_K;
  const uint16_t* P_V;
  uint16_t* k_lat;
  uint16_t* v_lat;
  int32_t* seq_lens;
  uint32_t* dev_status;
  int B, Hkv, T, d, rK, rV, L_max;
};

constexpr int kMaxSmemPerBlock = 232448;  // 227 KB opt-in dynamic shared memory (sm_100)

uint32_t decode_split_smem_bytes(int NW, int nstage, int G_T, int d, int rK, int rV);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_compress(const CompressArgs& a, cudaStream_t stream);

}  // namespace stief
