// decode_mode_paged_q8.cu -- the decode kernel's instantiations for int8 caches in page pools
// (codes and fp32 row scales per pool row, tiles addressed through a block table).
#include "decode_kernel.cuh"

namespace stief {

cudaError_t launch_decode_paged_q8(const DecodeArgs& a, cudaStream_t stream) {
  return launch_mode<kModePagedQ8>(a, stream);
}

}  // namespace stief
