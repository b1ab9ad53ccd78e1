// decode_mode_paged.cu -- the decode kernel's instantiations for paged caches (tiles addressed through a block table).
#include "decode_kernel.cuh"

namespace stief {

cudaError_t launch_decode_paged(const DecodeArgs& a, cudaStream_t stream) {
  return launch_mode<kModePaged>(a, stream);
}

}  // namespace stief
