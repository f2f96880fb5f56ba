// decode_kc.cu -- the decode attention kernel instantiated for K caches whose
// keys are quantized per channel over token groups (the KIVI-combined
// quantizer), with fp16 and bf16 caches; a translation unit of its own so that
// the builds run in parallel.
#include "decode_warp.cuh"

namespace gear {
cudaError_t decode_warp_launch_kc(const DecodeMaps& maps, const DecodeArgs& a, cudaStream_t st) {
  if (a.dtype == GEAR_F16) return launch_bits_kc<__half>(maps, a, st);
  if (a.dtype == GEAR_BF16) return launch_bits_kc<__nv_bfloat16>(maps, a, st);
  return cudaErrorInvalidValue;
}
}  // namespace gear
