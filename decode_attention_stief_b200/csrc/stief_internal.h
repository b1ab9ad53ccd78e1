// stief_internal.h -- argument blocks and launch entry points shared between the
// C-ABI host code (stief_api.cu) and the kernel files.  Not a public header.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "stief.h"

namespace stief {

// One column piece of the key cache: keys are fetched by 2-D TMA tensor copies in
// pieces 64, 32 or 16 columns wide, each with the matching 128-, 64- or 32-byte
// shared-memory swizzle (widths decrease along the row).
struct KeyPiece {
  int x;         // first column (a multiple of 16)
  int width;     // 64, 32 or 16 columns
  int smem_off;  // byte offset inside a key slot
  int map;       // index into DecodeArgs::tmk
};

// Everything the decode kernel needs, validated by the host code.  Passed as a
// __grid_constant__ parameter so the tensor maps can be addressed in place.
struct DecodeArgs {
  CUtensorMap tmk[3];  // key-cache maps for piece widths 64, 32, 16 (those in use)
  KeyPiece kp[4];
  int npieces;
  const uint16_t* q;
  const uint16_t* P_K;
  const uint16_t* P_V;
  const uint16_t* k_lat;
  const uint16_t* v_lat;
  const int32_t* seq_lens;
  uint16_t* out;
  uint32_t* ws_cnt;  // [units] split tickets; zero between calls
  float* ws_part;    // [units * S * G_T][rV + 4] partial states: o~[rV], m, l, 0, 0
  uint32_t* dev_status;
  int B, Hq, Hkv, G, G_T, qsub, d, rK, rV, L_max, S;
  int npairs;     // K-warp / V-warp pairs per CTA (4 or 8)
  int nstage;     // shared-memory stages per pair
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

uint32_t decode_smem_bytes(int NW, int nstage, int G_T, int d, int rK, int rV);

// 2-D tiled TMA tensor map over a row-major bf16 matrix [rows][cols] (row stride in
// bytes), boxes of box_cols x box_rows with the given swizzle.  Host only.
bool encode_tiled_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                          uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows,
                          CUtensorMapSwizzle swizzle);

struct CompressTcArgs;
uint32_t compress_tc_smem_bytes(int rK, int rV);

// Validates a decode call and fills everything in `a` except the workspace pointers
// (split count, group tiling, CTA configuration, key tensor maps).  Host only.
stief_status plan_decode(DecodeArgs& a, const uint16_t* q, const uint16_t* P_K,
                         const uint16_t* P_V, const uint16_t* k_lat, const uint16_t* v_lat,
                         const int32_t* seq_lens, uint16_t* out, int B, int Hq, int Hkv, int d,
                         int rK, int rV, int L_max, int max_seq_len, int num_splits,
                         uint32_t* dev_status);

// Decode workspace layout: `units` = B * Hkv * qsub ticket counters (uint32, padded to
// 256 bytes), then units * G_T * splits partial states of (rV + 4) floats.
inline size_t decode_ws_counter_bytes(size_t units) { return (units * 4u + 255u) / 256u * 256u; }
inline size_t decode_ws_bytes(size_t units, int G_T, int splits, int rV) {
  return decode_ws_counter_bytes(units) + units * (size_t)G_T * splits * (size_t)(rV + 4) * 4u;
}
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);

// Pairs per CTA and stages per pair for the decode kernel: at least 3 stages per pair
// (one tile in the K-warp, one in the V-warp, one in flight) where shared memory allows,
// 8 pairs unless G_T == 8 (whose 8-pair build would spill), else the widest that fits.
inline bool choose_decode_config(int G_T, int d, int rK, int rV, int* npairs, int* nstage) {
  const int first = G_T == 8 ? 4 : 8;
  for (int min_ns : {3, 2})
    for (int np : {first, 4})
      for (int ns = 4; ns >= min_ns; --ns)
        if (decode_smem_bytes(np, ns, G_T, d, rK, rV) <= (uint32_t)kMaxSmemPerBlock) {
          *npairs = np;
          *nstage = ns;
          return true;
        }
  return false;
}
cudaError_t launch_compress(const CompressArgs& a, cudaStream_t stream);

}  // namespace stief
