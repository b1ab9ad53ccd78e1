// decode_kernels.cu -- dispatch of a planned decode call to the kernel instantiation of its
// mode (each mode's instantiations live in their own translation unit, decode_mode_*.cu).
#include "decode_kernel.cuh"

namespace stief {

uint32_t decode_smem_bytes(int nwarps, int nstage, int rK, int rV, int tile, int code) {
  return decode_smem_layout(nwarps, nstage, rK, rV, tile, code).total;
}

uint32_t decode_region_bytes(int nwarps, int nstage, int rK, int rV, int tile, int code) {
  return decode_smem_layout(nwarps, nstage, rK, rV, tile, code).region_bytes;
}

// the latent decode, paged, int8 and joint-value caches are their own instantiations, so their
// branches cost the contiguous path nothing (a runtime flag cost it 0.5-0.8 us per launch)
cudaError_t launch_decode(const DecodeArgs& planned, cudaStream_t stream) {
  DecodeArgs a = planned;
  // right after a compress of this library the new rows may still be in flight when this
  // kernel starts: no cache tile is requested before the dependency wait then
  a.early = take_stream_compress_mark(a.device, stream) ? 0 : 1;
  if (a.block_table != nullptr && a.q8 != 0 && a.latent == 0 && a.q4 == 0 && a.append == 0)
    return launch_decode_paged_q8(a, stream);  // int8 codes in page pools
  if ((a.latent != 0) + (a.block_table != nullptr) + (a.q8 != 0) + (a.q4 != 0) > 1)
    return cudaErrorInvalidValue;  // the other modes do not combine
  if (a.q4 != 0 && a.append != 0) return cudaErrorInvalidValue;  // no 4-bit fused step
  if (a.joint_v) {
    if (a.block_table != nullptr || a.q8 != 0 || a.q4 != 0 || a.append != 0) return cudaErrorInvalidValue;
    return a.latent ? launch_decode_latent_joint_v(a, stream) : launch_decode_joint_v(a, stream);
  }
  if (a.latent) return launch_decode_latent(a, stream);
  if (a.block_table) return launch_decode_paged(a, stream);
  if (a.q8 && a.append) {
    // the int8 fused step writes a cache row that the next decode in the stream would read
    // before its dependency wait (int8 tiles get no second read of that row): note it
    const cudaError_t e = launch_decode_q8_append(a, stream);
    if (e == cudaSuccess) mark_stream_compress(a.device, stream, true);
    return e;
  }
  if (a.q8) return launch_decode_q8(a, stream);
  if (a.q4) return launch_decode_q4(a, stream);
  return launch_decode_plain(a, stream);
}

}  // namespace stief
