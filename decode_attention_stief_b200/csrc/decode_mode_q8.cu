// decode_mode_q8.cu -- the decode kernel's instantiations for int8 caches (codes and fp32 row scales).
#include "decode_kernel.cuh"

namespace stief {

cudaError_t launch_decode_q8(const DecodeArgs& a, cudaStream_t stream) {
  return launch_mode<kModeQ8>(a, stream);
}

}  // namespace stief
