// stief_internal.h -- argument blocks and launch entry points shared between the
// C-ABI host code (stief_api.cu) and the kernel files.  Not a public header.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "stief.h"

namespace stief {

// One column piece of a bf16 matrix fetched by 2-D TMA tensor copies: matrices of
// rank r are read in pieces 64, 32 or 16 columns wide (widths decreasing along the
// row), each landing with the matching 128-, 64- or 32-byte shared-memory swizzle,
// so that eight rows of one 16-byte column chunk sit in eight different bank groups.
struct Piece {
  int x;         // first column (a multiple of 16)
  int width;     // 64, 32 or 16 columns
  int smem_off;  // byte offset of the piece inside the tile
  int map;       // index into DecodeArgs::maps
};
struct PieceSet {
  Piece p[4];
  int n;
};

// Everything the decode kernel needs, validated by the host code.  Passed as a
// __grid_constant__ parameter so the tensor maps can be addressed in place.
struct DecodeArgs {
  CUtensorMap maps[12];  // per (matrix, piece width) in use
  int nmaps;
  PieceSet pk, pv;       // key / value cache tiles of 32 rows
  PieceSet ppk, ppv;     // P_K / P_V of d rows
  const uint16_t* q;
  const int32_t* seq_lens;
  uint16_t* out;
  // append path (stief_append_decode): the new token's rows, the caches and lengths it writes
  int append;
  const uint16_t* k_new;  // [B][Hkv][d]
  const uint16_t* v_new;  // [B][Hkv][d]
  uint16_t* k_lat_w;
  uint16_t* v_lat_w;
  int32_t* seq_lens_w;
  uint32_t* ws_seq;  // [B] per-sequence finish tickets; zero between calls
  uint32_t* ws_cnt;  // [units] split tickets; zero between calls
  // Split partial states, in one of two forms over the same bytes:
  //  - ticket merge: float [units * S * G_T][rV + 4]: o~[rV] (latent), m, l, 0, 0
  //  - tagged merge: uint64 [units * S * G_T][rV + 2]: o~[rV], m, l as tagged words (value,
  //    tag 1 when written); every word is zero between calls
  float* ws_part;
  uint64_t* ws_words;
  int merge_tagged;  // 1: the tagged merge (the grid fits on the GPU at once), 0: tickets
  uint32_t* dev_status;
  int B, Hq, Hkv, G, G_T, qsub, d, rK, rV, L_max, S;
  int max_seq_len;  // host bound of seq_lens; the splits partition [0, S * chunk)
  int chunk;        // tokens per split, a multiple of the 32-token tile
  int tile;         // tokens per tile: 32, or 64 when rK + rV <= 96
  int nwarps;       // consumer warps per CTA, each streaming its own tiles
  int nstage;       // shared-memory stages per warp
  float qscale;     // log2(e) / sqrt(d), applied to q . P_K
  int device;       // current device at planning time (host bookkeeping only)
  int latent;       // latent decode: q holds q~ [B][Hq][rK], out is o~ [B][Hq][rV], no bases
  // paged caches: [num_pages][Hkv][page_size][r] pools addressed through block_table
  // [B][max_pages] (null for a contiguous cache; L_max is then max_pages * page_size)
  const int32_t* block_table;
  int max_pages, page_size, num_pages;
  // int8 caches: k_lat / v_lat hold int8 codes [rows][r] and these the fp32 row scales;
  // 4-bit caches (q4): two codes per byte, [rows][r / 2], with the same row scales
  int q8;
  int q4;
  int joint_v;     // values: one row per (sequence, token) shared by the KV heads
  // 1: the contiguous bf16 and latent modes request each warp's first tile before the
  // dependency wait; 0 when the library's previous launch in the stream was a compress (its
  // length kernel lets the next kernel start while the new rows are still being written)
  int early;
  const float* k_scale;
  const float* v_scale;
  // int8 fused step: the scale arrays the new token's row scales are written to
  float* k_scale_w;
  float* v_scale_w;
#ifdef STIEF_TEST_HOOKS
  // test build only: bytes added to the setup barrier's expected count that no copy delivers,
  // so that its phase never completes and the waits for it run out (0: off)
  uint32_t test_stall_bytes;
#endif
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
  int device;  // current device (host bookkeeping only)
  // paged caches, as in DecodeArgs (block_table null: contiguous [B][Hkv][L_max] rows)
  const int32_t* block_table;
  int max_pages, page_size, num_pages;
  // int8 caches: k_lat / v_lat take int8 codes and these the fp32 row scales (null: bf16);
  // with q4 the codes are 4-bit, two per byte ([rows][r / 2])
  float* k_scale;
  float* v_scale;
  int q4;
#ifdef STIEF_TEST_HOOKS
  // test build only: bytes added to the first copy's expected count in every CTA (half) of
  // the tensor-core projections, which no copy delivers, so that the waits for it run out
  uint32_t test_stall_bytes;
#endif
};

constexpr int kMaxSmemPerBlock = 232448;  // 227 KB opt-in dynamic shared memory (sm_100)
constexpr int kMaxDevices = 64;

// The current device, its SM count and whether it is sm_100 (queried once per device).
// Returns false if the CUDA runtime cannot answer.  Host only.
bool query_device(int* dev, int* sms, bool* sm100);

// A kernel's dynamic shared-memory limit, raised once per device to the largest size
// requested so far (cudaFuncSetAttribute is not repeated on every launch).
struct SmemLimit {
  std::atomic<int> set[kMaxDevices] = {};
  cudaError_t ensure(const void* kern, int dev, int bytes) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    int cur = set[dev].load(std::memory_order_relaxed);
    if (bytes <= cur) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    while (bytes > cur && !set[dev].compare_exchange_weak(cur, bytes)) {
    }
    return cudaSuccess;
  }
};

// code: 0 bf16 cache, 1 int8 codes, 2 4-bit codes
uint32_t decode_smem_bytes(int nwarps, int nstage, int rK, int rV, int tile, int code = 0);
// Bytes of the region (rings, then the warp-merge and split-merge staging) in that layout.
uint32_t decode_region_bytes(int nwarps, int nstage, int rK, int rV, int tile, int code = 0);

// 2-D tiled TMA tensor map over a row-major bf16 matrix [rows][cols] (row stride in
// bytes), boxes of box_cols x box_rows with the given swizzle.  Host only.
bool encode_tiled_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                          uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows,
                          CUtensorMapSwizzle swizzle);

struct CompressTcArgs;
uint32_t compress_tc_smem_bytes(int rK, int rV);

// Validates a decode call and fills everything in `a` except the workspace pointers
// (split count, group tiling, CTA configuration, key tensor maps).  Host only.
// With `latent`, q is q~ [B][Hq][rK], out is o~ [B][Hq][rV] and P_K, P_V are unused (may be
// NULL): no base tensor maps are planned.  With a block table, k_lat / v_lat are page pools
// [num_pages][Hkv][page_size][r] and L_max is the capacity max_pages * page_size.  With row
// scales (k_scale, v_scale), k_lat / v_lat are int8 codes [B][Hkv][L_max][r].
stief_status plan_decode(DecodeArgs& a, const uint16_t* q, const uint16_t* P_K,
                         const uint16_t* P_V, const uint16_t* k_lat, const uint16_t* v_lat,
                         const int32_t* seq_lens, uint16_t* out, int B, int Hq, int Hkv, int d,
                         int rK, int rV, int L_max, int max_seq_len, int num_splits,
                         uint32_t* dev_status, bool latent = false,
                         const int32_t* block_table = nullptr, int max_pages = 0,
                         int page_size = 0, int num_pages = 0, const float* k_scale = nullptr,
                         const float* v_scale = nullptr, bool joint_v = false, bool q4 = false);

// Decode workspace layout: `units` = B * Hkv * qsub split-ticket counters, then B sequence
// tickets (uint32, padded together to 256 bytes), then units * G_T * splits partial-state
// records of (d + 2) 8-byte words (a tagged record uses r_V + 2 <= d + 2 words, a ticket
// record r_V + 4 <= 2 d + 4 floats).
inline size_t decode_ws_counter_bytes(size_t units, size_t B) {
  return ((units + B) * 4u + 255u) / 256u * 256u;
}
inline size_t decode_ws_bytes(size_t units, size_t B, int G_T, int splits, int d) {
  return decode_ws_counter_bytes(units, B) + units * (size_t)G_T * splits * (size_t)(d + 2) * 8u;
}
// Bytes of the tagged partial-state words a call with this plan writes (the prefix of the
// record area that must be zero when it starts).
inline size_t decode_ws_tagged_bytes(size_t units, int G_T, int splits, int rV) {
  return units * (size_t)G_T * splits * (size_t)(rV + 2) * 8u;
}
// Shared-memory bytes the merging CTA of the tagged merge stages the records in: its heads'
// records as [nh][rV + 2 columns][splits padded to a multiple of 4] floats, where
// nh <= ceil(G_T / S) heads are merged by one CTA.
inline size_t decode_tagged_stage_bytes(int G_T, int splits, int rV) {
  const int nh = (G_T + splits - 1) / splits;
  return 4u * (size_t)nh * (rV + 2) * (size_t)((splits + 3) & ~3);
}
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);

// Per (device, stream): whether the library's last launch there wrote cache rows that the next
// decode could request before its dependency wait: a compress (whose length kernel lets its
// dependent start early) or an int8 fused step.  Those mark their stream; a decode reads and
// clears the mark (it then requests no cache tile before its dependency wait); the joint
// compress's CUDA-core path, whose kernels do not let dependents start early, clears it.
// Host only.
void mark_stream_compress(int device, cudaStream_t s, bool marked);
bool take_stream_compress_mark(int device, cudaStream_t s);

// Tokens per tile: 64 for small ranks (an SM sustains a roughly fixed number of tiles per
// microsecond, so small tiles would leave the memory system idle), 32 otherwise.
inline int choose_decode_tile(int rK, int rV) { return rK <= 64 && rV <= 64 && rK + rV <= 96 ? 64 : 32; }
// int8 caches: rows take half the bytes, so 64-token tiles whenever both ranks are <= 64.
inline int choose_decode_tile_q8(int rK, int rV) { return rK <= 64 && rV <= 64 ? 64 : 32; }

// Consumer warps per CTA and stages per warp for the decode kernel: 8 warps with as many
// stages (up to 8) as shared memory allows, fewer warps only when 8 cannot have two each.
// Grids of more than one wave (one split, more units than SMs) run two CTAs per SM with a
// smaller ring, so that one CTA's prologue and epilogue overlap the other's streaming (at
// batch 64 x 8 KV heads x 4096 tokens: 87.8 instead of 100.7 us per launch).  Two CTAs fit
// when each takes at most half of the SM's 228 KB less the 1 KB the system reserves per CTA,
// and when 2 x (warps + producer) x 32 threads x 168 registers fit in 64 K: at most five
// consumer warps.  Fewer than four consumer warps per CTA is not worth it.
constexpr int kPairSmemPerBlock = 233472 / 2 - 1024;
constexpr int kPairMaxConsumerWarps = 5;
inline bool choose_decode_config_pair(int rK, int rV, int tile, int* nwarps, int* nstage,
                                      int code = 0) {
  for (int nw = kPairMaxConsumerWarps; nw >= 4; --nw)
    for (int ns = 4; ns >= 2; --ns)
      if (decode_smem_bytes(nw, ns, rK, rV, tile, code) <= (uint32_t)kPairSmemPerBlock) {
        *nwarps = nw;
        *nstage = ns;
        return true;
      }
  return false;
}
inline bool choose_decode_config(int rK, int rV, int tile, int* nwarps, int* nstage,
                                 int code = 0) {
  for (int nw = 8; nw >= 2; --nw)
    for (int ns = 8; ns >= 2; --ns)
      if (decode_smem_bytes(nw, ns, rK, rV, tile, code) <= (uint32_t)kMaxSmemPerBlock) {
        *nwarps = nw;
        *nstage = ns;
        return true;
      }
  return false;
}
cudaError_t launch_compress(const CompressArgs& a, cudaStream_t stream);
#ifdef STIEF_TEST_HOOKS
// test build only: the stall the next decode launches are planned with (see DecodeArgs)
uint32_t test_stall_bytes();
#endif
// Joint value latents: keys per head into k_lat, the values of all KV heads of a token
// through P_V = P_VJ [Hkv*d][rV] into v_lat = v_joint [B][L_max][rV]; then the lengths.
cudaError_t launch_compress_joint(const CompressArgs& a, cudaStream_t stream);
// The length update seq_lens[b] += T of a compress (contiguous or paged rows), launched as a
// programmatic dependent of the projection; it lets its own dependents start early.
cudaError_t launch_seq_lens(const CompressArgs& a, cudaStream_t stream);
// The tcgen05 joint-value projection of prefill-sized chunks (d = 128), and whether its
// shared memory (the whole joint basis plus a ring of at least two input chunks) fits.
bool compress_joint_tc_fits(int Hkv, int rK, int rV);
cudaError_t launch_compress_joint_tc(const CompressArgs& a, cudaStream_t stream);

}  // namespace stief
