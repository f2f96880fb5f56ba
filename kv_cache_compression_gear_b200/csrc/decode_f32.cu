// decode_f32.cu -- the decode attention kernel instantiated for float caches
// (one translation unit per dtype, so that the builds run in parallel).
#include "decode_warp.cuh"

namespace gear {
cudaError_t decode_warp_launch_f32(const DecodeMaps& maps, const DecodeArgs& a, cudaStream_t st) {
  return launch_bits<float>(maps, a, st);
}
}  // namespace gear
