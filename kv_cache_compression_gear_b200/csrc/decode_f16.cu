// decode_f16.cu -- the decode attention kernel instantiated for __half caches
// (one translation unit per dtype, so that the builds run in parallel).
#include "decode_warp.cuh"

namespace gear {
cudaError_t decode_warp_launch_f16(const DecodeMaps& maps, const DecodeArgs& a, cudaStream_t st) {
  return launch_bits<__half>(maps, a, st);
}
}  // namespace gear
