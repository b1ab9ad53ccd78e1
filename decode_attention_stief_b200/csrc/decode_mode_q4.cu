// decode_mode_q4.cu -- the decode kernel's instantiations for 4-bit caches (two codes per byte,
// fp32 row scales).
#include "decode_kernel.cuh"

namespace stief {

cudaError_t launch_decode_q4(const DecodeArgs& a, cudaStream_t stream) {
  return launch_mode<kModeQ4>(a, stream);
}

}  // namespace stief
