// decode_mode_plain.cu -- the decode kernel's instantiations for the contiguous bf16 cache.
#include "decode_kernel.cuh"

namespace stief {

cudaError_t launch_decode_plain(const DecodeArgs& a, cudaStream_t stream) {
  return launch_mode<kModePlain>(a, stream);
}

}  // namespace stief
