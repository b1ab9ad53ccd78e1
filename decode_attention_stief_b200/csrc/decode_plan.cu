// decode_plan.cu -- host-side planning shared by the two decode entry points:
// argument checks, split count, CTA configuration and the key-cache tensor maps.
#include <cmath>
#include <cstdint>
#include <atomic>
#include <map>
#include <mutex>
#include <utility>

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

// Tensor maps are pure functions of (base, r, rows, box rows, width); decoding the same
// layer's cache over and over re-uses them from this table instead of re-encoding (an
// encode costs on the order of a microsecond of host time per map).
struct MapKey {
  const void* base;
  uint64_t rows;
  int r, box_rows, width;
  bool operator==(const MapKey& o) const {
    return base == o.base && rows == o.rows && r == o.r && box_rows == o.box_rows && width == o.width;
  }
};
constexpr int kMapCacheSlots = 1024;
struct MapSlot {
  MapKey key;
  CUtensorMap map;
  bool used;
};
std::mutex g_map_mu;
MapSlot g_map_cache[kMapCacheSlots];

bool cached_map(CUtensorMap* out, const void* base, int r, uint64_t rows, int box_rows, int width) {
  const MapKey key{base, rows, r, box_rows, width};
  uint64_t h = reinterpret_cast<uintptr_t>(base) * 0x9E3779B97F4A7C15ull;
  h ^= rows * 0xC2B2AE3D27D4EB4Full + (uint64_t)r * 131 + (uint64_t)box_rows * 7 + (uint64_t)width;
  h ^= h >> 29;
  MapSlot& slot = g_map_cache[h % kMapCacheSlots];
  {
    std::lock_guard<std::mutex> lock(g_map_mu);
    if (slot.used && slot.key == key) {
      *out = slot.map;
      return true;
    }
  }
  const CUtensorMapSwizzle sw = width == 64   ? CU_TENSOR_MAP_SWIZZLE_128B
                                : width == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : width == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                              : CU_TENSOR_MAP_SWIZZLE_NONE;
  if (!encode_tiled_bf16_2d(out, base, (uint64_t)r, rows, (uint64_t)r * 2u, (uint32_t)width,
                            (uint32_t)box_rows, sw))
    return false;
  std::lock_guard<std::mutex> lock(g_map_mu);
  slot.key = key;
  slot.map = *out;
  slot.used = true;
  return true;
}

// Column pieces of a matrix r 16-bit columns wide (r a multiple of 8): widths 64, 64, 32,
// 16, 8 taken in that order while they fit, each with its own tensor map (one per width,
// shared by the pieces of that width) over `base` viewed as [rows][r] 16-bit elements, boxes
// of width x box_rows, swizzled 128, 64 or 32 bytes (the 8-wide piece, 16 bytes, is not
// swizzled).  Pieces are stacked in shared memory in the same order.  A bf16 matrix of rank r
// is r columns; an int8 matrix of rank r is viewed as r / 2 columns (the copy moves bytes).
bool plan_pieces(DecodeArgs& a, int* nmaps, PieceSet& ps, const void* base, int r, uint64_t rows,
                 int box_rows) {
  int map_of_width[4] = {-1, -1, -1, -1};  // for 64, 32, 16, 8
  int x = 0, off = 0;
  ps.n = 0;
  for (int w : {64, 64, 32, 16, 8}) {
    if (r - x < w) continue;
    const int wi = w == 64 ? 0 : w == 32 ? 1 : w == 16 ? 2 : 3;
    if (map_of_width[wi] < 0) {
      if (*nmaps >= 12) return false;
      if (!cached_map(&a.maps[*nmaps], base, r, rows, box_rows, w)) return false;
      map_of_width[wi] = (*nmaps)++;
    }
    if (ps.n >= 3) return false;
    Piece& p = ps.p[ps.n++];
    p.x = x;
    p.width = w;
    p.smem_off = off;
    p.map = map_of_width[wi];
    x += w;
    off += box_rows * w * 2;
  }
  return x == r;
}

struct DevInfo {
  int sms;
  bool sm100;
  bool ok;
};
DevInfo g_dev_info[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

#ifdef STIEF_TEST_HOOKS
std::atomic<uint32_t> g_test_stall{0};
#endif

}  // namespace

#ifdef STIEF_TEST_HOOKS
uint32_t test_stall_bytes() { return g_test_stall.load(); }
#endif

namespace {
std::mutex g_mark_mu;
std::map<std::pair<int, cudaStream_t>, bool> g_compress_mark;  // (device, stream) -> marked
}  // namespace

void mark_stream_compress(int device, cudaStream_t s, bool marked) {
  std::lock_guard<std::mutex> lock(g_mark_mu);
  if (marked) g_compress_mark[{device, s}] = true;
  else g_compress_mark.erase({device, s});
}

bool take_stream_compress_mark(int device, cudaStream_t s) {
  std::lock_guard<std::mutex> lock(g_mark_mu);
  return g_compress_mark.erase({device, s}) != 0;
}

bool query_device(int* dev_out, int* sms, bool* sm100) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::call_once(g_dev_once[dev], [dev] {
    int major = 0, minor = 0, n = 0;
    DevInfo di{0, false, false};
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
      di = DevInfo{n, major == 10 && minor == 0, true};
    g_dev_info[dev] = di;
  });
  *dev_out = dev;
  *sms = g_dev_info[dev].sms;
  *sm100 = g_dev_info[dev].sm100;
  return g_dev_info[dev].ok;
}

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
                         uint32_t* dev_status, bool latent, const int32_t* block_table,
                         int max_pages, int page_size, int num_pages, const float* k_scale,
                         const float* v_scale, bool joint_v, bool q4) {
  const bool q8 = k_scale != nullptr && !q4;  // int8 codes
  if (q4 && (k_scale == nullptr || rK % 32 != 0 || rV % 32 != 0)) return STIEF_ERR_INVALID_ARG;
  if (joint_v && (block_table || q8 || q4)) return STIEF_ERR_INVALID_ARG;
  const int code = q8 ? 1 : q4 ? 2 : 0;  // the stage layout's code form
  if (!q || !k_lat || !v_lat || !seq_lens || !out) return STIEF_ERR_INVALID_ARG;
  if (!latent && (!P_K || !P_V)) return STIEF_ERR_INVALID_ARG;
  if (B < 1 || B > 65535 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Hq / Hkv > 64)
    return STIEF_ERR_INVALID_ARG;
  if (d != 128 || !rank_ok(rK) || !rank_ok(rV) || L_max < 1 || max_seq_len < 0)
    return STIEF_ERR_INVALID_ARG;
  if (max_seq_len > L_max) return STIEF_ERR_CAPACITY;
  const int smax = stief_decode_max_splits(max_seq_len);
  if (num_splits < 0 || num_splits > smax) return STIEF_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_lat) || !aligned16(v_lat) || !aligned16(out))
    return STIEF_ERR_ALIGNMENT;
  if (!latent && (!aligned16(P_K) || !aligned16(P_V))) return STIEF_ERR_ALIGNMENT;
  // rows of the cache tensors: contiguous [B][Hkv][L_max], or pools [num_pages][Hkv][page_size]
  const uint64_t rows = block_table ? (uint64_t)num_pages * Hkv * page_size : (uint64_t)B * Hkv * L_max;
  if (rows >= (1ull << 31)) return STIEF_ERR_INVALID_ARG;  // TMA row coordinates are int32
  // joint values: one row per (sequence, token), [B][L_max][rV], read by every KV head
  const uint64_t vrows = joint_v ? (uint64_t)B * L_max : rows;

  int dev = 0, sms = 0;
  bool sm100 = false;
  if (!query_device(&dev, &sms, &sm100)) return STIEF_ERR_CUDA;
  if (!sm100) return STIEF_ERR_UNSUPPORTED_DEVICE;
  a.device = dev;
  a.latent = latent ? 1 : 0;
  a.block_table = block_table;
  a.max_pages = max_pages;
  a.page_size = page_size;
  a.num_pages = num_pages;
  a.joint_v = joint_v ? 1 : 0;

  a.q = q;
  a.seq_lens = seq_lens;
  a.out = out;
  // the caches' base pointers (the tiles come through the tensor maps; the fused step writes
  // its new rows here, and the kernel reads the row just below each length again here)
  a.k_lat_w = const_cast<uint16_t*>(k_lat);
  a.v_lat_w = const_cast<uint16_t*>(v_lat);
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
  a.max_seq_len = max_seq_len;
  // tokens per split: the split's share rounded up to whole 32-token tiles, so that only
  // the last tile of a sequence can be partial
  a.tile = (q8 || q4) ? choose_decode_tile_q8(rK, rV) : choose_decode_tile(rK, rV);
  a.chunk = ((max_seq_len + a.S - 1) / a.S + a.tile - 1) / a.tile * a.tile;
  a.qscale = (float)(1.4426950408889634 / std::sqrt((double)d));
  const long long units = (long long)B * a.Hkv * a.qsub;
  const bool pair = a.S == 1 && units > sms &&
                    choose_decode_config_pair(rK, rV, a.tile, &a.nwarps, &a.nstage, code);
  if (!pair && !choose_decode_config(rK, rV, a.tile, &a.nwarps, &a.nstage, code))
    return STIEF_ERR_INVALID_ARG;
  // Split merge: through tagged words when the whole grid is on the GPU at once (one CTA per
  // SM at most, so every split of a unit runs while its merging CTA reads their records) and
  // the merging CTA's staging fits its shared memory; otherwise by tickets (no CTA waits for
  // another).
  a.merge_tagged = 0;
  if (a.S > 1 && (long long)a.S * units <= sms &&
      decode_tagged_stage_bytes(a.G_T, a.S, rV) <=
          decode_region_bytes(a.nwarps, a.nstage, rK, rV, a.tile, code))
    a.merge_tagged = 1;

  int nmaps = 0;
  const uint64_t prow = (uint64_t)Hkv * d;
  a.q8 = q8 ? 1 : 0;
  a.q4 = q4 ? 1 : 0;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  // the caches' column pieces (int8 codes: rows of r bytes, moved as r / 2 16-bit columns;
  // 4-bit codes: r / 2 bytes, r / 4 columns)
  const int kc = q8 ? rK / 2 : q4 ? rK / 4 : rK, vc = q8 ? rV / 2 : q4 ? rV / 4 : rV;
  if (!plan_pieces(a, &nmaps, a.pk, k_lat, kc, rows, a.tile) ||
      !plan_pieces(a, &nmaps, a.pv, v_lat, vc, vrows, a.tile))
    return STIEF_ERR_CUDA;
  if (!latent && (!plan_pieces(a, &nmaps, a.ppk, P_K, rK, prow, d) ||
                  !plan_pieces(a, &nmaps, a.ppv, P_V, rV, prow, d)))
    return STIEF_ERR_CUDA;
  a.nmaps = nmaps;
#ifdef STIEF_TEST_HOOKS
  a.test_stall_bytes = test_stall_bytes();
#endif
  return STIEF_OK;
}

}  // namespace stief

#ifdef STIEF_TEST_HOOKS
// Test build only (libstief_testhooks.so, used by the timeout tests; not part of the public
// header): every decode planned after this call waits for `bytes` more on its setup barrier
// than any copy delivers, and every tensor-core compress launched after it for `bytes` more on
// each CTA's (half's) first copy, so their bounded waits run out (0 turns it off).  The bytes
// must be a multiple of 16.
extern "C" STIEF_API void stief_test_set_stall(uint32_t bytes) { stief::g_test_stall.store(bytes); }
#endif
