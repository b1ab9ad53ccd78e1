// decode_mode_joint_v.cu -- the decode kernel's instantiations for joint value latents, full output.
#include "decode_kernel.cuh"

namespace stief {

cudaError_t launch_decode_joint_v(const DecodeArgs& a, cudaStream_t stream) {
  return launch_mode<kModeJointV>(a, stream);
}

}  // namespace stief
