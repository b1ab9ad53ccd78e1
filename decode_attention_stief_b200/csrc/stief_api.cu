// stief_api.cu -- the C ABI declared in include/stief.h: argument checking,
// split planning, workspace sizing and kernel launches.  Host code only.
#include <cmath>
#include <cstdint>
#include <cstring>

#include <cuda_runtime.h>

#include "stief.h"
#include "stief_internal.h"

namespace {

constexpr int kHeadDim = 128;          // the only supported d
constexpr int kMinTokensPerSplit = 128;
constexpr int kMaxSplits = 512;
constexpr int kMaxGroup = 64;          // largest Hq / Hkv

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool rank_ok(int r) { return r >= 16 && r <= kHeadDim && (r % 16) == 0; }

int group_tile(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8; }

stief_status device_check(int* dev) {
  int sms = 0;
  bool sm100 = false;
  if (!stief::query_device(dev, &sms, &sm100)) return STIEF_ERR_CUDA;
  if (!sm100) return STIEF_ERR_UNSUPPORTED_DEVICE;
  return STIEF_OK;
}

// Common decode shape checks (host only, no CUDA call).
stief_status check_decode_shape(int B, int Hq, int Hkv, int d, int rK, int rV, int L_max,
                                int max_seq_len) {
  if (B < 1 || B > 65535 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Hq / Hkv > kMaxGroup)
    return STIEF_ERR_INVALID_ARG;
  if (d != kHeadDim || !rank_ok(rK) || !rank_ok(rV)) return STIEF_ERR_INVALID_ARG;
  if (L_max < 1 || max_seq_len < 0) return STIEF_ERR_INVALID_ARG;
  if (max_seq_len > L_max) return STIEF_ERR_CAPACITY;
  return STIEF_OK;
}

// A paged cache: pools [num_pages][Hkv][page_size][r] and a block table [B][max_pages]
// (null for the contiguous layout).
struct Paging {
  const int32_t* block_table = nullptr;
  int num_pages = 0, page_size = 0, max_pages = 0;
};

constexpr int kPageQuantum = 64;  // page sizes are multiples of the largest decode tile
constexpr int kQ8RowQuantum = 64;  // int8 caches: L_max is a multiple of the largest tile,
                                   // so a tile's scale copy never passes a head's rows

// Host checks of a paged cache; on success *capacity = max_pages * page_size tokens.
stief_status check_paging(const Paging& pg, int Hkv, int* capacity) {
  if (!pg.block_table) return STIEF_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(pg.block_table) & 3u) != 0) return STIEF_ERR_ALIGNMENT;
  if (pg.page_size < kPageQuantum || pg.page_size % kPageQuantum != 0 || pg.num_pages < 1 ||
      pg.max_pages < 1 || Hkv < 1)
    return STIEF_ERR_INVALID_ARG;
  const long long cap = (long long)pg.max_pages * pg.page_size;
  const long long rows = (long long)pg.num_pages * Hkv * pg.page_size;
  if (cap > 0x7fffffffLL || rows >= (1LL << 31)) return STIEF_ERR_INVALID_ARG;
  *capacity = (int)cap;
  return STIEF_OK;
}

}  // namespace

extern "C" {

const char* stief_status_string(stief_status s) {
  switch (s) {
    case STIEF_OK: return "STIEF_OK";
    case STIEF_ERR_INVALID_ARG: return "STIEF_ERR_INVALID_ARG";
    case STIEF_ERR_ALIGNMENT: return "STIEF_ERR_ALIGNMENT";
    case STIEF_ERR_CAPACITY: return "STIEF_ERR_CAPACITY";
    case STIEF_ERR_WORKSPACE: return "STIEF_ERR_WORKSPACE";
    case STIEF_ERR_CUDA: return "STIEF_ERR_CUDA";
    case STIEF_ERR_DEVICE_STATUS: return "STIEF_ERR_DEVICE_STATUS";
    case STIEF_ERR_UNSUPPORTED_DEVICE: return "STIEF_ERR_UNSUPPORTED_DEVICE";
  }
  return "STIEF_ERR_UNKNOWN";
}

int stief_decode_max_splits(int max_seq_len) {
  if (max_seq_len < 0) return 0;
  int s = (max_seq_len + kMinTokensPerSplit - 1) / kMinTokensPerSplit;
  if (s < 1) s = 1;
  if (s > kMaxSplits) s = kMaxSplits;
  return s;
}

int stief_decode_auto_splits(int B, int Hq, int Hkv, int max_seq_len, int num_sms) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || max_seq_len < 0 || num_sms < 1) return 0;
  const int G = Hq / Hkv;
  const int qsub = (G + group_tile(G) - 1) / group_tile(G);
  const long long units = (long long)B * Hkv * qsub;
  // one split CTA per SM: split only while there are fewer units than SMs
  long long s = units >= num_sms ? 1 : num_sms / units;
  const int smax = stief_decode_max_splits(max_seq_len);
  if (s > smax) s = smax;
  if (s < 1) s = 1;
  return (int)s;
}

size_t stief_decode_workspace_bytes(int B, int Hq, int Hkv, int rV, int max_seq_len) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || !rank_ok(rV) || max_seq_len < 0) return 0;
  const int G = Hq / Hkv;
  const int G_T = group_tile(G);
  const int qsub = (G + G_T - 1) / G_T;
  const size_t units = (size_t)B * Hkv * qsub;
  return stief::decode_ws_bytes(units, (size_t)B, G_T, stief_decode_max_splits(max_seq_len), kHeadDim);
}

}  // extern "C"

namespace {

stief_status compress_common(const uint16_t* k_new, const uint16_t* v_new, const uint16_t* P_K,
                             const uint16_t* P_V, uint16_t* k_lat, uint16_t* v_lat,
                             int32_t* seq_lens, int B, int Hkv, int T, int d, int rK, int rV,
                             int L_max, uint32_t* dev_status, stief_stream_t stream,
                             const Paging& pg, float* k_scale = nullptr,
                             float* v_scale = nullptr, bool q4 = false) {
  if (!k_new || !v_new || !P_K || !P_V || !k_lat || !v_lat || !seq_lens) return STIEF_ERR_INVALID_ARG;
  if (pg.block_table) {
    const stief_status st = check_paging(pg, Hkv, &L_max);
    if (st != STIEF_OK) return st;
  }
  if (B < 1 || Hkv < 1 || T < 0 || d != kHeadDim || !rank_ok(rK) || !rank_ok(rV) || L_max < 1)
    return STIEF_ERR_INVALID_ARG;
  if (T > L_max) return STIEF_ERR_CAPACITY;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(P_K) || !aligned16(P_V) ||
      !aligned16(k_lat) || !aligned16(v_lat))
    return STIEF_ERR_ALIGNMENT;
  if (T == 0) return STIEF_OK;
  int dev = 0;
  stief_status st = device_check(&dev);
  if (st != STIEF_OK) return st;
  stief::CompressArgs a{};
  a.device = dev;
  a.k_new = k_new;
  a.v_new = v_new;
  a.P_K = P_K;
  a.P_V = P_V;
  a.k_lat = k_lat;
  a.v_lat = v_lat;
  a.seq_lens = seq_lens;
  a.dev_status = dev_status;
  a.B = B;
  a.Hkv = Hkv;
  a.T = T;
  a.d = d;
  a.rK = rK;
  a.rV = rV;
  a.L_max = L_max;
  a.block_table = pg.block_table;
  a.max_pages = pg.max_pages;
  a.page_size = pg.page_size;
  a.num_pages = pg.num_pages;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.q4 = q4 ? 1 : 0;
  if (stief::launch_compress(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return STIEF_ERR_CUDA;
  return STIEF_OK;
}

}  // namespace

extern "C" {

stief_status stief_compress_append(const uint16_t* k_new, const uint16_t* v_new,
                                   const uint16_t* P_K, const uint16_t* P_V, uint16_t* k_lat,
                                   uint16_t* v_lat, int32_t* seq_lens, int B, int Hkv, int T,
                                   int d, int rK, int rV, int L_max, uint32_t* dev_status,
                                   stief_stream_t stream) {
  return compress_common(k_new, v_new, P_K, P_V, k_lat, v_lat, seq_lens, B, Hkv, T, d, rK, rV,
                         L_max, dev_status, stream, Paging{});
}

stief_status stief_compress_append_q8(const uint16_t* k_new, const uint16_t* v_new,
                                      const uint16_t* P_K, const uint16_t* P_V, int8_t* k_q,
                                      int8_t* v_q, float* k_s, float* v_s, int32_t* seq_lens,
                                      int B, int Hkv, int T, int d, int rK, int rV, int L_max,
                                      uint32_t* dev_status, stief_stream_t stream) {
  if (!k_s || !v_s) return STIEF_ERR_INVALID_ARG;
  if (L_max % kQ8RowQuantum != 0) return STIEF_ERR_INVALID_ARG;
  if (!aligned16(k_s) || !aligned16(v_s)) return STIEF_ERR_ALIGNMENT;
  return compress_common(k_new, v_new, P_K, P_V, reinterpret_cast<uint16_t*>(k_q),
                         reinterpret_cast<uint16_t*>(v_q), seq_lens, B, Hkv, T, d, rK, rV, L_max,
                         dev_status, stream, Paging{}, k_s, v_s);
}

stief_status stief_compress_append_q8_paged(const uint16_t* k_new, const uint16_t* v_new,
                                            const uint16_t* P_K, const uint16_t* P_V,
                                            int8_t* k_pages, int8_t* v_pages, float* k_s_pages,
                                            float* v_s_pages, const int32_t* block_table,
                                            int32_t* seq_lens, int B, int Hkv, int T, int d,
                                            int rK, int rV, int num_pages, int page_size,
                                            int max_pages, uint32_t* dev_status,
                                            stief_stream_t stream) {
  Paging pg;
  pg.block_table = block_table;
  pg.num_pages = num_pages;
  pg.page_size = page_size;
  pg.max_pages = max_pages;
  if (!block_table || !k_s_pages || !v_s_pages) return STIEF_ERR_INVALID_ARG;
  if (!aligned16(k_s_pages) || !aligned16(v_s_pages)) return STIEF_ERR_ALIGNMENT;
  return compress_common(k_new, v_new, P_K, P_V, reinterpret_cast<uint16_t*>(k_pages),
                         reinterpret_cast<uint16_t*>(v_pages), seq_lens, B, Hkv, T, d, rK, rV, 0,
                         dev_status, stream, pg, k_s_pages, v_s_pages);
}

stief_status stief_compress_append_q4(const uint16_t* k_new, const uint16_t* v_new,
                                      const uint16_t* P_K, const uint16_t* P_V, uint8_t* k_q,
                                      uint8_t* v_q, float* k_s, float* v_s, int32_t* seq_lens,
                                      int B, int Hkv, int T, int d, int rK, int rV, int L_max,
                                      uint32_t* dev_status, stief_stream_t stream) {
  if (!k_s || !v_s) return STIEF_ERR_INVALID_ARG;
  if (L_max % kQ8RowQuantum != 0 || rK % 32 != 0 || rV % 32 != 0) return STIEF_ERR_INVALID_ARG;
  if (!aligned16(k_s) || !aligned16(v_s)) return STIEF_ERR_ALIGNMENT;
  return compress_common(k_new, v_new, P_K, P_V, reinterpret_cast<uint16_t*>(k_q),
                         reinterpret_cast<uint16_t*>(v_q), seq_lens, B, Hkv, T, d, rK, rV, L_max,
                         dev_status, stream, Paging{}, k_s, v_s, true);
}

stief_status stief_compress_append_paged(const uint16_t* k_new, const uint16_t* v_new,
                                         const uint16_t* P_K, const uint16_t* P_V,
                                         uint16_t* k_pages, uint16_t* v_pages,
                                         const int32_t* block_table, int32_t* seq_lens, int B,
                                         int Hkv, int T, int d, int rK, int rV, int num_pages,
                                         int page_size, int max_pages, uint32_t* dev_status,
                                         stief_stream_t stream) {
  Paging pg;
  pg.block_table = block_table;
  pg.num_pages = num_pages;
  pg.page_size = page_size;
  pg.max_pages = max_pages;
  if (!block_table) return STIEF_ERR_INVALID_ARG;
  return compress_common(k_new, v_new, P_K, P_V, k_pages, v_pages, seq_lens, B, Hkv, T, d, rK,
                         rV, 0, dev_status, stream, pg);
}

namespace {

// Shared body of stief_decode_attention and stief_append_decode.
stief_status decode_common(const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                           const uint16_t* P_K, const uint16_t* P_V, uint16_t* k_lat,
                           uint16_t* v_lat, int32_t* seq_lens, uint16_t* out, void* workspace,
                           size_t workspace_bytes, int B, int Hq, int Hkv, int d, int rK, int rV,
                           int L_max, int max_seq_len, int num_splits, uint32_t* dev_status,
                           stief_stream_t stream, bool append, bool latent = false,
                           const Paging& pg = Paging{}, const float* k_scale = nullptr,
                           const float* v_scale = nullptr, bool joint_v = false,
                           bool q4 = false) {
  // cheap host checks first, so argument errors never touch CUDA
  if (!q || !k_lat || !v_lat || !seq_lens || !out) return STIEF_ERR_INVALID_ARG;
  if (pg.block_table) {  // paged: the capacity is max_pages * page_size tokens
    const stief_status sp = check_paging(pg, Hkv, &L_max);
    if (sp != STIEF_OK) return sp;
  }
  if (!latent && (!P_K || !P_V)) return STIEF_ERR_INVALID_ARG;
  if (append && (!k_new || !v_new)) return STIEF_ERR_INVALID_ARG;
  stief_status st = check_decode_shape(B, Hq, Hkv, d, rK, rV, L_max, max_seq_len);
  if (st != STIEF_OK) return st;
  const int smax = stief_decode_max_splits(max_seq_len);
  if (num_splits < 0 || num_splits > smax) return STIEF_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_lat) || !aligned16(v_lat) || !aligned16(out) ||
      !aligned16(workspace))
    return STIEF_ERR_ALIGNMENT;
  if (!latent && (!aligned16(P_K) || !aligned16(P_V))) return STIEF_ERR_ALIGNMENT;
  if (append && (!aligned16(k_new) || !aligned16(v_new))) return STIEF_ERR_ALIGNMENT;
  const size_t need = stief_decode_workspace_bytes(B, Hq, Hkv, rV, max_seq_len);
  if (!workspace || workspace_bytes < need) return STIEF_ERR_WORKSPACE;

  stief::DecodeArgs a{};
  st = stief::plan_decode(a, q, P_K, P_V, k_lat, v_lat, seq_lens, out, B, Hq, Hkv, d, rK, rV,
                          L_max, max_seq_len, num_splits, dev_status, latent, pg.block_table,
                          pg.max_pages, pg.page_size, pg.num_pages, k_scale, v_scale, joint_v,
                          q4);
  if (st != STIEF_OK) return st;
  a.append = append ? 1 : 0;
  a.k_new = k_new;
  a.v_new = v_new;
  a.k_lat_w = k_lat;
  a.v_lat_w = v_lat;
  a.seq_lens_w = seq_lens;
  // the int8 fused step writes the new token's row scales (the caller's arrays are writable)
  a.k_scale_w = const_cast<float*>(k_scale);
  a.v_scale_w = const_cast<float*>(v_scale);
  // counters at the start (split tickets, then sequence tickets), then the partial states
  // laid out for the split count used
  const size_t units = (size_t)B * Hkv * a.qsub;
  a.ws_cnt = static_cast<uint32_t*>(workspace);
  a.ws_seq = a.ws_cnt + units;
  a.ws_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                       stief::decode_ws_counter_bytes(units, (size_t)B));
  a.ws_words = reinterpret_cast<uint64_t*>(a.ws_part);
  if (stief::launch_decode(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return STIEF_ERR_CUDA;
  return STIEF_OK;
}

}  // namespace

stief_status stief_decode_attention(const uint16_t* q, const uint16_t* P_K, const uint16_t* P_V,
                                    const uint16_t* k_lat, const uint16_t* v_lat,
                                    const int32_t* seq_lens, uint16_t* out, void* workspace,
                                    size_t workspace_bytes, int B, int Hq, int Hkv, int d, int rK,
                                    int rV, int L_max, int max_seq_len, int num_splits,
                                    uint32_t* dev_status, stief_stream_t stream) {
  // the caches and lengths are only read on this path
  return decode_common(q, nullptr, nullptr, P_K, P_V, const_cast<uint16_t*>(k_lat),
                       const_cast<uint16_t*>(v_lat), const_cast<int32_t*>(seq_lens), out,
                       workspace, workspace_bytes, B, Hq, Hkv, d, rK, rV, L_max, max_seq_len,
                       num_splits, dev_status, stream, false);
}

stief_status stief_append_decode(const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                                 const uint16_t* P_K, const uint16_t* P_V, uint16_t* k_lat,
                                 uint16_t* v_lat, int32_t* seq_lens, uint16_t* out,
                                 void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                                 int d, int rK, int rV, int L_max, int max_seq_len,
                                 int num_splits, uint32_t* dev_status, stief_stream_t stream) {
  return decode_common(q, k_new, v_new, P_K, P_V, k_lat, v_lat, seq_lens, out, workspace,
                       workspace_bytes, B, Hq, Hkv, d, rK, rV, L_max, max_seq_len, num_splits,
                       dev_status, stream, true);
}

stief_status stief_decode_latent(const uint16_t* q_lat, const uint16_t* k_lat,
                                 const uint16_t* v_lat, const int32_t* seq_lens, uint16_t* out_lat,
                                 void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                                 int d, int rK, int rV, int L_max, int max_seq_len, int num_splits,
                                 uint32_t* dev_status, stief_stream_t stream) {
  return decode_common(q_lat, nullptr, nullptr, nullptr, nullptr, const_cast<uint16_t*>(k_lat),
                       const_cast<uint16_t*>(v_lat), const_cast<int32_t*>(seq_lens), out_lat,
                       workspace, workspace_bytes, B, Hq, Hkv, d, rK, rV, L_max, max_seq_len,
                       num_splits, dev_status, stream, false, true);
}

stief_status stief_compress_append_joint_v(const uint16_t* k_new, const uint16_t* v_new,
                                           const uint16_t* P_K, const uint16_t* P_VJ,
                                           uint16_t* k_lat, uint16_t* v_joint, int32_t* seq_lens,
                                           int B, int Hkv, int T, int d, int rK, int rV,
                                           int L_max, uint32_t* dev_status,
                                           stief_stream_t stream) {
  if (!k_new || !v_new || !P_K || !P_VJ || !k_lat || !v_joint || !seq_lens)
    return STIEF_ERR_INVALID_ARG;
  if (B < 1 || B > 65535 || Hkv < 1 || Hkv > 65534 || T < 0 || d != kHeadDim || !rank_ok(rK) ||
      !rank_ok(rV) || L_max < 1)
    return STIEF_ERR_INVALID_ARG;
  if (T > L_max) return STIEF_ERR_CAPACITY;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(P_K) || !aligned16(P_VJ) ||
      !aligned16(k_lat) || !aligned16(v_joint))
    return STIEF_ERR_ALIGNMENT;
  if (T == 0) return STIEF_OK;
  int dev = 0;
  const stief_status st = device_check(&dev);
  if (st != STIEF_OK) return st;
  stief::CompressArgs a{};
  a.device = dev;
  a.k_new = k_new;
  a.v_new = v_new;
  a.P_K = P_K;
  a.P_V = P_VJ;
  a.k_lat = k_lat;
  a.v_lat = v_joint;
  a.seq_lens = seq_lens;
  a.dev_status = dev_status;
  a.B = B;
  a.Hkv = Hkv;
  a.T = T;
  a.d = d;
  a.rK = rK;
  a.rV = rV;
  a.L_max = L_max;
  if (stief::launch_compress_joint(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return STIEF_ERR_CUDA;
  return STIEF_OK;
}

stief_status stief_decode_attention_joint_v(const uint16_t* q, const uint16_t* P_K,
                                            const uint16_t* P_VJ, const uint16_t* k_lat,
                                            const uint16_t* v_joint, const int32_t* seq_lens,
                                            uint16_t* out, void* workspace,
                                            size_t workspace_bytes, int B, int Hq, int Hkv,
                                            int d, int rK, int rV, int L_max, int max_seq_len,
                                            int num_splits, uint32_t* dev_status,
                                            stief_stream_t stream) {
  return decode_common(q, nullptr, nullptr, P_K, P_VJ, const_cast<uint16_t*>(k_lat),
                       const_cast<uint16_t*>(v_joint), const_cast<int32_t*>(seq_lens), out,
                       workspace, workspace_bytes, B, Hq, Hkv, d, rK, rV, L_max, max_seq_len,
                       num_splits, dev_status, stream, false, false, Paging{}, nullptr, nullptr,
                       true);
}

stief_status stief_decode_latent_joint_v(const uint16_t* q_lat, const uint16_t* k_lat,
                                         const uint16_t* v_joint, const int32_t* seq_lens,
                                         uint16_t* out_lat, void* workspace,
                                         size_t workspace_bytes, int B, int Hq, int Hkv, int d,
                                         int rK, int rV, int L_max, int max_seq_len,
                                         int num_splits, uint32_t* dev_status,
                                         stief_stream_t stream) {
  return decode_common(q_lat, nullptr, nullptr, nullptr, nullptr, const_cast<uint16_t*>(k_lat),
                       const_cast<uint16_t*>(v_joint), const_cast<int32_t*>(seq_lens), out_lat,
                       workspace, workspace_bytes, B, Hq, Hkv, d, rK, rV, L_max, max_seq_len,
                       num_splits, dev_status, stream, false, true, Paging{}, nullptr, nullptr,
                       true);
}

stief_status stief_decode_attention_q8(const uint16_t* q, const uint16_t* P_K,
                                       const uint16_t* P_V, const int8_t* k_q, const int8_t* v_q,
                                       const float* k_s, const float* v_s,
                                       const int32_t* seq_lens, uint16_t* out, void* workspace,
                                       size_t workspace_bytes, int B, int Hq, int Hkv, int d,
                                       int rK, int rV, int L_max, int max_seq_len,
                                       int num_splits, uint32_t* dev_status,
                                       stief_stream_t stream) {
  if (!k_s || !v_s) return STIEF_ERR_INVALID_ARG;
  if (L_max % kQ8RowQuantum != 0) return STIEF_ERR_INVALID_ARG;
  if (!aligned16(k_s) || !aligned16(v_s)) return STIEF_ERR_ALIGNMENT;
  return decode_common(q, nullptr, nullptr, P_K, P_V,
                       reinterpret_cast<uint16_t*>(const_cast<int8_t*>(k_q)),
                       reinterpret_cast<uint16_t*>(const_cast<int8_t*>(v_q)),
                       const_cast<int32_t*>(seq_lens), out, workspace, workspace_bytes, B, Hq, Hkv,
                       d, rK, rV, L_max, max_seq_len, num_splits, dev_status, stream, false, false,
                       Paging{}, k_s, v_s);
}

stief_status stief_append_decode_q8(const uint16_t* q, const uint16_t* k_new,
                                    const uint16_t* v_new, const uint16_t* P_K,
                                    const uint16_t* P_V, int8_t* k_q, int8_t* v_q, float* k_s,
                                    float* v_s, int32_t* seq_lens, uint16_t* out, void* workspace,
                                    size_t workspace_bytes, int B, int Hq, int Hkv, int d, int rK,
                                    int rV, int L_max, int max_seq_len, int num_splits,
                                    uint32_t* dev_status, stief_stream_t stream) {
  if (!k_s || !v_s) return STIEF_ERR_INVALID_ARG;
  if (L_max % kQ8RowQuantum != 0) return STIEF_ERR_INVALID_ARG;
  if (!aligned16(k_s) || !aligned16(v_s)) return STIEF_ERR_ALIGNMENT;
  return decode_common(q, k_new, v_new, P_K, P_V, reinterpret_cast<uint16_t*>(k_q),
                       reinterpret_cast<uint16_t*>(v_q), seq_lens, out, workspace,
                       workspace_bytes, B, Hq, Hkv, d, rK, rV, L_max, max_seq_len, num_splits,
                       dev_status, stream, true, false, Paging{}, k_s, v_s);
}

stief_status stief_decode_attention_q8_paged(const uint16_t* q, const uint16_t* P_K,
                                             const uint16_t* P_V, const int8_t* k_pages,
                                             const int8_t* v_pages, const float* k_s_pages,
                                             const float* v_s_pages, const int32_t* block_table,
                                             const int32_t* seq_lens, uint16_t* out,
                                             void* workspace, size_t workspace_bytes, int B,
                                             int Hq, int Hkv, int d, int rK, int rV, int num_pages,
                                             int page_size, int max_pages, int max_seq_len,
                                             int num_splits, uint32_t* dev_status,
                                             stief_stream_t stream) {
  Paging pg;
  pg.block_table = block_table;
  pg.num_pages = num_pages;
  pg.page_size = page_size;
  pg.max_pages = max_pages;
  if (!block_table || !k_s_pages || !v_s_pages) return STIEF_ERR_INVALID_ARG;
  if (!aligned16(k_s_pages) || !aligned16(v_s_pages)) return STIEF_ERR_ALIGNMENT;
  return decode_common(q, nullptr, nullptr, P_K, P_V,
                       reinterpret_cast<uint16_t*>(const_cast<int8_t*>(k_pages)),
                       reinterpret_cast<uint16_t*>(const_cast<int8_t*>(v_pages)),
                       const_cast<int32_t*>(seq_lens), out, workspace, workspace_bytes, B, Hq, Hkv,
                       d, rK, rV, 0, max_seq_len, num_splits, dev_status, stream, false, false, pg,
                       k_s_pages, v_s_pages);
}

stief_status stief_decode_attention_q4(const uint16_t* q, const uint16_t* P_K,
                                       const uint16_t* P_V, const uint8_t* k_q, const uint8_t* v_q,
                                       const float* k_s, const float* v_s,
                                       const int32_t* seq_lens, uint16_t* out, void* workspace,
                                       size_t workspace_bytes, int B, int Hq, int Hkv, int d,
                                       int rK, int rV, int L_max, int max_seq_len,
                                       int num_splits, uint32_t* dev_status,
                                       stief_stream_t stream) {
  if (!k_s || !v_s) return STIEF_ERR_INVALID_ARG;
  if (L_max % kQ8RowQuantum != 0 || rK % 32 != 0 || rV % 32 != 0) return STIEF_ERR_INVALID_ARG;
  if (!aligned16(k_s) || !aligned16(v_s)) return STIEF_ERR_ALIGNMENT;
  return decode_common(q, nullptr, nullptr, P_K, P_V,
                       reinterpret_cast<uint16_t*>(const_cast<uint8_t*>(k_q)),
                       reinterpret_cast<uint16_t*>(const_cast<uint8_t*>(v_q)),
                       const_cast<int32_t*>(seq_lens), out, workspace, workspace_bytes, B, Hq, Hkv,
                       d, rK, rV, L_max, max_seq_len, num_splits, dev_status, stream, false, false,
                       Paging{}, k_s, v_s, false, true);
}

stief_status stief_decode_attention_paged(const uint16_t* q, const uint16_t* P_K,
                                          const uint16_t* P_V, const uint16_t* k_pages,
                                          const uint16_t* v_pages, const int32_t* block_table,
                                          const int32_t* seq_lens, uint16_t* out, void* workspace,
                                          size_t workspace_bytes, int B, int Hq, int Hkv, int d,
                                          int rK, int rV, int num_pages, int page_size,
                                          int max_pages, int max_seq_len, int num_splits,
                                          uint32_t* dev_status, stief_stream_t stream) {
  Paging pg;
  pg.block_table = block_table;
  pg.num_pages = num_pages;
  pg.page_size = page_size;
  pg.max_pages = max_pages;
  if (!block_table) return STIEF_ERR_INVALID_ARG;
  return decode_common(q, nullptr, nullptr, P_K, P_V, const_cast<uint16_t*>(k_pages),
                       const_cast<uint16_t*>(v_pages), const_cast<int32_t*>(seq_lens), out,
                       workspace, workspace_bytes, B, Hq, Hkv, d, rK, rV, 0, max_seq_len,
                       num_splits, dev_status, stream, false, false, pg);
}

stief_status stief_append_decode_paged(const uint16_t* q, const uint16_t* k_new,
                                       const uint16_t* v_new, const uint16_t* P_K,
                                       const uint16_t* P_V, uint16_t* k_pages, uint16_t* v_pages,
                                       const int32_t* block_table, int32_t* seq_lens,
                                       uint16_t* out, void* workspace, size_t workspace_bytes,
                                       int B, int Hq, int Hkv, int d, int rK, int rV,
                                       int num_pages, int page_size, int max_pages,
                                       int max_seq_len, int num_splits, uint32_t* dev_status,
                                       stief_stream_t stream) {
  Paging pg;
  pg.block_table = block_table;
  pg.num_pages = num_pages;
  pg.page_size = page_size;
  pg.max_pages = max_pages;
  if (!block_table) return STIEF_ERR_INVALID_ARG;
  return decode_common(q, k_new, v_new, P_K, P_V, k_pages, v_pages, seq_lens, out, workspace,
                       workspace_bytes, B, Hq, Hkv, d, rK, rV, 0, max_seq_len, num_splits,
                       dev_status, stream, true, false, pg);
}

stief_status stief_read_device_status(const uint32_t* dev_status, uint32_t* value,
                                      stief_stream_t stream) {
  if (!dev_status || !value) return STIEF_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(value, dev_status, sizeof(uint32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return STIEF_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return STIEF_ERR_CUDA;
  return *value == 0 ? STIEF_OK : STIEF_ERR_DEVICE_STATUS;
}

}  // extern "C"
