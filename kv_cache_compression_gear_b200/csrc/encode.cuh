// encode.cuh -- argument block and host entry of the GEAR encoder kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gear {

// Up to kMaxBatch same-shaped tensors (for example the K and V of a layer)
// are encoded by one launch of each kernel. Unit u of the batch is unit
// u % Uper of tensor u / Uper.
constexpr int kMaxBatch = 16;

// Per-unit "Z slab" that E2 writes for E3 (bytes): the fp32 rows of Z
// [128 channels][16 ranks], then S_g [4][16] floats with the power-of-two
// scale of the images and its inverse, then the tensor-core operand images.
constexpr int kSlabRows = 0;
constexpr int kSlabS = 8192;          // 64 floats, then down, up (272 bytes in all)
constexpr int kSlabSBytes = 272;
constexpr int kSlabImg = 9216;        // X Z parts (3 x 4 KB at most), then C Z parts (2 x 16 KB at most)
constexpr int kZSlab = kSlabImg + 3 * 4096 + 2 * 16384;

struct EncodeTensor {
  const void* kv;    // input rows [Uper][n][128], cache dtype
  uint32_t* codes;   // the tensor's cache arrays
  float* meta;
  uint8_t* oidx;
  void* oval;
  void* lfac;
  float* rfac;
};

struct EncodeArgs {
  int32_t nt, Uper;  // tensors, units per tensor
  int32_t U, n;      // U = nt * Uper units of n tokens each
  int32_t dtype;     // gear_dtype
  // codec
  int32_t bits, g, k, r, T;
  uint64_t seed;
  // destination in the caches: tokens [t_off, t_off + n) of block `blk`
  int32_t t_off, blk, e_blk;
  uint32_t one_bits;     // 0x3F800000 (1.0f), kept in a register by the kernels
  int32_t n_max, nblk_max, W, G, r_max;
  int32_t meta_f16;      // scale and zero stored as binary16
  int32_t ch;            // per-channel key groups of g tokens (meta per token-group slot)
  int32_t ch_slots;      // token-group slots per unit of the cache (ch)
  int32_t slot0;         // slot of this block's first token group (ch)
  // workspace: partial Grams [U][maxc][128][128] and Z slabs [U][kZSlab bytes] (E3 operands)
  float* gram;
  float* zbuf;
  // tiling of E1
  int32_t tpu;           // 128-token tiles per unit
  int64_t total_tiles;   // U * tpu
  int32_t grid_e1;       // persistent CTAs of E1
  int32_t maxc;          // partial-Gram slots per unit
  int32_t e3_tpc;        // consecutive 128-token tiles per CTA of the low-rank pass (16-bit inputs)
  EncodeTensor ten[kMaxBatch];
};

int encode_grid(const EncodeArgs& a, int num_sms);
int encode_maxc(int64_t total_tiles, int grid, int tpu);
cudaError_t encode_launch(EncodeArgs a, int num_sms, cudaStream_t st);

}  // namespace gear
