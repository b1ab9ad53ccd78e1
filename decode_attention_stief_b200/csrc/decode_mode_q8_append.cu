// decode_mode_q8_append.cu -- the decode kernel's instantiations for the int8 fused step
// (append the new token's quantised rows, then decode over the int8 cache).
#include "decode_kernel.cuh"

namespace stief {

cudaError_t launch_decode_q8_append(const DecodeArgs& a, cudaStream_t stream) {
  return launch_mode<kModeQ8Append>(a, stream);
}

}  // namespace stief
