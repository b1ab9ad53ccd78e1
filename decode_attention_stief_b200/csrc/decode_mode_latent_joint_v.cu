// decode_mode_latent_joint_v.cu -- the decode kernel's instantiations for joint value latents, latent output.
#include "decode_kernel.cuh"

namespace stief {

cudaError_t launch_decode_latent_joint_v(const DecodeArgs& a, cudaStream_t stream) {
  return launch_mode<kModeLatentJointV>(a, stream);
}

}  // namespace stief
