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
// How.  The scratch is a file-scope __device__ array of kScratchBytes (8 MiB),
// laid out like the caller workspace of stief_decode_attention: split ticket
// counters first, then the partial states.
// Every GPU that loads this library holds one such array until the process
// exits.  Host code cannot use the array's name as a device address, so on the
// first call on each device (with that device current) the address is looked up
// with cudaGetSymbolAddress and cached; that first call should therefore happen
// before any stream capture.  All calls share the one array per device:
// concurrent calls whose kernels overlap on the GPU (different streams, or
// several host threads) race on it and must be serialised by the caller.  The
// array keeps the previous call's contents.  The ticket counters and the tagged
// words of the split merge must be zero when a call starts; a call that runs to
// completion leaves them so, but one that stopped early (a wait timeout) may not,
// and the caller cannot reach the array to clear it.  So every call zeroes the
// part it will use with cudaMemsetAsync on its stream before the launch (the
// partial states themselves are always written before they are read).  Sizes
// whose partial states do not fit are rejected with STIEF_ERR_WORKSPACE before
// anything is launched.  No cudaMalloc, cudaFree or allocating library routine
// is called.
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "stief.h"
#include "stief_internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;
using stief::kMaxDevices;

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

}  // namespace

extern "C" STIEF_API stief_status stief_decode_attention_noalloc(
    const uint16_t* q, const uint16_t* P_K, const uint16_t* P_V, const uint16_t* k_lat,
    const uint16_t* v_lat, const int32_t* seq_lens, uint16_t* out, int B, int Hq, int Hkv, int d,
    int rK, int rV, int L_max, int max_seq_len, int num_splits, uint32_t* dev_status,
    stief_stream_t stream) {
  stief::DecodeArgs a{};
  stief_status st = stief::plan_decode(a, q, P_K, P_V, k_lat, v_lat, seq_lens, out, B, Hq, Hkv, d,
                                       rK, rV, L_max, max_seq_len, num_splits, dev_status);
  if (st != STIEF_OK) return st;

  // ticket counters and the partial states of the split count actually used must fit
  const size_t units = (size_t)B * Hkv * a.qsub;
  if (stief::decode_ws_bytes(units, (size_t)B, a.G_T, a.S, a.d) > kScratchBytes)
    return STIEF_ERR_WORKSPACE;

  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != STIEF_OK) return st;
  a.ws_cnt = static_cast<uint32_t*>(scratch);
  a.ws_seq = a.ws_cnt + units;
  a.ws_part = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) +
                                       stief::decode_ws_counter_bytes(units, (size_t)B));
  a.ws_words = reinterpret_cast<uint64_t*>(a.ws_part);
  // The ticket counters (and the tagged words of the split merge) must be zero when the
  // kernel starts.  A call that completes leaves them so, but one that stopped early (a wait
  // timeout) may not, and the caller cannot reach this array to clear it: zero them here, in
  // stream order, before every launch (a memset, not an allocation).
  size_t clear = stief::decode_ws_counter_bytes(units, (size_t)B);
  if (a.merge_tagged) clear += stief::decode_ws_tagged_bytes(units, a.G_T, a.S, a.rV);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, clear, s) != cudaSuccess) return STIEF_ERR_CUDA;
  if (stief::launch_decode(a, s) != cudaSuccess) return STIEF_ERR_CUDA;
  return STIEF_OK;
}

#ifdef STIEF_TEST_HOOKS
// Test build only: the device address of this library's scratch array on the current device,
// so that a test can plant stale counters in it (the public calls never expose it).
extern "C" STIEF_API stief_status stief_test_noalloc_scratch(void** ptr, size_t* bytes) {
  if (!ptr || !bytes) return STIEF_ERR_INVALID_ARG;
  *bytes = kScratchBytes;
  return scratch_address(ptr);
}
#endif
