// decode_plan.cu -- host-side planning shared by the two decode entry points:
// argument checks, split count, CTA configuration and the key-cache tensor maps.
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "stief.h"
#include "stief_internal.h"

namespace stief {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool rank_ok(int r) { return r >= 16 && r <= 128 && (r % 16) == 0; }
int group_tile(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8; }

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D view of the key cache: [B*Hkv*L_max rows][rK columns] bf16, boxes of 32 rows x width.
bool encode_key_map(CUtensorMap* map, const uint16_t* k_lat, int rK, uint64_t rows, int width) {
  const CUtensorMapSwizzle sw = width == 64   ? CU_TENSOR_MAP_SWIZZLE_128B
                                : width == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                              : CU_TENSOR_MAP_SWIZZLE_32B;
  return encode_tiled_bf16_2d(map, k_lat, (uint64_t)rK, rows, (uint64_t)rK * 2u, (uint32_t)width,
                              32u, sw);
}

}  // namespace

bool encode_tiled_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                          uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows,
                          CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)row_stride_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

stief_status plan_decode(DecodeArgs& a, const uint16_t* q, const uint16_t* P_K,
                         const uint16_t* P_V, const uint16_t* k_lat, const uint16_t* v_lat,
                         const int32_t* seq_lens, uint16_t* out, int B, int Hq, int Hkv, int d,
                         int rK, int rV, int L_max, int max_seq_len, int num_splits,
                         uint32_t* dev_status) {
  if (!q || !P_K || !P_V || !k_lat || !v_lat || !seq_lens || !out) return STIEF_ERR_INVALID_ARG;
  if (B < 1 || B > 65535 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Hq / Hkv > 64)
    return STIEF_ERR_INVALID_ARG;
  if (d != 128 || !rank_ok(rK) || !rank_ok(rV) || L_max < 1 || max_seq_len < 0)
    return STIEF_ERR_INVALID_ARG;
  if (max_seq_len > L_max) return STIEF_ERR_CAPACITY;
  const int smax = stief_decode_max_splits(max_seq_len);
  if (num_splits < 0 || num_splits > smax) return STIEF_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(P_K) || !aligned16(P_V) || !aligned16(k_lat) ||
      !aligned16(v_lat) || !aligned16(out))
    return STIEF_ERR_ALIGNMENT;
  const uint64_t rows = (uint64_t)B * Hkv * L_max;
  if (rows >= (1ull << 31)) return STIEF_ERR_INVALID_ARG;  // TMA row coordinates are int32

  int dev = 0, major = 0, minor = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return STIEF_ERR_CUDA;
  if (major != 10 || minor != 0) return STIEF_ERR_UNSUPPORTED_DEVICE;

  a.q = q;
  a.P_K = P_K;
  a.P_V = P_V;
  a.k_lat = k_lat;
  a.v_lat = v_lat;
  a.seq_lens = seq_lens;
  a.out = out;
  a.dev_status = dev_status;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.G_T = group_tile(a.G);
  a.qsub = (a.G + a.G_T - 1) / a.G_T;
  a.d = d;
  a.rK = rK;
  a.rV = rV;
  a.L_max = L_max;
  a.S = num_splits > 0 ? num_splits : stief_decode_auto_splits(B, Hq, Hkv, max_seq_len, sms);
  a.qscale = (float)(1.4426950408889634 / std::sqrt((double)d));
  a.pdl_first = false;
  if (!choose_decode_config(a.G_T, d, rK, rV, &a.npairs, &a.nstage)) return STIEF_ERR_INVALID_ARG;

  // key pieces: widths 64, 32, 16 in decreasing order (rK is a multiple of 16)
  int map_of_width[3] = {-1, -1, -1};  // for 64, 32, 16
  int nmaps = 0, x = 0, off = 0;
  a.npieces = 0;
  for (int w : {64, 64, 32, 16}) {
    if (rK - x < w) continue;
    const int wi = w == 64 ? 0 : w == 32 ? 1 : 2;
    if (map_of_width[wi] < 0) {
      if (!encode_key_map(&a.tmk[nmaps], k_lat, rK, rows, w)) return STIEF_ERR_CUDA;
      map_of_width[wi] = nmaps++;
    }
    KeyPiece& kp = a.kp[a.npieces++];
    kp.x = x;
    kp.width = w;
    kp.smem_off = off;
    kp.map = map_of_width[wi];
    x += w;
    off += 32 * w * 2;
  }
  if (x != rK) return STIEF_ERR_INVALID_ARG;
  return STIEF_OK;
}

}  // namespace stief
