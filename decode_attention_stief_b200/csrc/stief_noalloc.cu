// stief_noalloc.cu -- stief_decode_attention_noalloc: the decode step without a
// caller-provided workspace and without any device allocation.
//
// Who needs it.  Some callers cannot obtain device memory at the point where they
// decode.  A serving engine typically reserves almost all of HBM for its KV-cache
// pool at start-up, so a later cudaMalloc either fails or eats into that pool; a
// host framework's custom-operator interface may hand a kernel only its input and
// output buffers, with no hook for temporary memory; and a latency-critical decode
// loop may not tolerate cudaMalloc, which can synchronise the device.  For them
// this entry point keeps the per-split partial softmax states in a fixed array of
// device memory that belongs to the library itself.
//
// How.  The scratch is a file-scope __device__ array of kScratchBytes (8 MiB).
// Every GPU that loads this library holds one such array until the process
// exits.  Host code cannot use the array's name as a device address, so on the
// first call on each device (with that device current) the address is looked up
// with cudaGetSymbolAddress and cached; that first call should therefore happen
// before any stream capture.  All calls share the one array per device:
// concurrent calls whose kernels overlap on the GPU (different streams, or
// several host threads) race on it and must be serialised by the caller.  The
// array keeps the previous call's contents; nothing in it needs to start at zero
// because every partial state is written by the split kernel before the combine
// kernel reads it.  Sizes whose partial states do not fit are rejected with
// STIEF_ERR_WORKSPACE before anything is launched.  No cudaMalloc, cudaFree or
// allocating library routine is called.
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/stief.h"
#include "stief_internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) float g_decode_scratch[kScratchBytes / sizeof(float)];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once per device).
stief_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return STIEF_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return STIEF_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return STIEF_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool rank_ok(int r) { return r >= 16 && r <= 128 && (r % 16) == 0; }
int group_tile(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8; }

}  // namespace

extern "C" STIEF_API stief_status stief_decode_attention_noalloc(
    const uint16_t* q, const uint16_t* P_K, const uint16_t* P_V, const uint16_t* k_lat,
    const uint16_t* v_lat, const int32_t* seq_lens, uint16_t* out, int B, int Hq, int Hkv, int d,
    int rK, int rV, int L_max, int max_seq_len, int num_splits, uint32_t* dev_status,
    stief_stream_t stream) {
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

  int dev = 0, major = 0, minor = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return STIEF_ERR_CUDA;
  if (major != 10 || minor != 0) return STIEF_ERR_UNSUPPORTED_DEVICE;

  stief::DecodeArgs a{};
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

  // the partial states of the split count actually used must fit the static scratch
  const size_t parts = (size_t)B * Hkv * a.qsub * a.G_T * a.S;
  if (parts * (size_t)(rV + 2) * sizeof(float) > kScratchBytes) return STIEF_ERR_WORKSPACE;

  void* scratch = nullptr;
  stief_status st = scratch_address(&scratch);
  if (st != STIEF_OK) return st;
  a.ws_o = static_cast<float*>(scratch);
  a.ws_ml = a.ws_o + parts * rV;

  a.nwarps = 0;
  for (int nw : {8, 4}) {
    for (int ns = 4; ns >= 2; --ns) {
      if (stief::decode_split_smem_bytes(nw, ns, a.G_T, d, rK, rV) <= (uint32_t)stief::kMaxSmemPerBlock) {
        a.nwarps = nw;
        a.nstage = ns;
        break;
      }
    }
    if (a.nwarps) break;
  }
  if (!a.nwarps) return STIEF_ERR_INVALID_ARG;
  if (stief::launch_decode(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return STIEF_ERR_CUDA;
  return STIEF_OK;
}
