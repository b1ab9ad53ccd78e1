// decode_mode_latent.cu -- the decode kernel's instantiations for the latent decode (q~ given, o~ returned).
#include "decode_kernel.cuh"

namespace stief {

cudaError_t launch_decode_latent(const DecodeArgs& a, cudaStream_t stream) {
  return launch_mode<kModeLatent>(a, stream);
}

}  // namespace stief
