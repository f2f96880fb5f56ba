// decode.cuh -- argument blocks of the GEAR decode-attention kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gear {

// One compressed tensor as the decode kernels see it.
struct CacheView {
  const uint32_t* codes;
  const float* meta;
  const uint8_t* oidx;
  const void* oval;
  const void* lfac;
  const float* rfac;
  const void* buf;
};

// Byte offsets of one tensor's 32-token tile in shared memory.
struct TileLayout {
  int32_t codes, meta, oidx, oval, lf, bytes;
};

struct DecodeArgs {
  CacheView K, V;
  int32_t dtype;          // cache dtype
  int32_t B, H, Hq, hq;   // hq = Hq / H query heads per kv head
  int32_t bits, g, G, W, k, r_max;
  int32_t n_max, nblk_max, n_b;
  int32_t n_comp, n_buf;
  int32_t blk0_len, blk0_rank, buffer_rank;
  float scale_log2;       // softmax scale * log2(e)
  const void* q;          // [B][Hq][128] cache dtype
  void* out;              // [B][Hq][128] out dtype
  int32_t out_dtype;
  float* part;            // [B][Hq][nsplit][130] partial (m, l, acc[128])
  int32_t chunk;          // compressed tokens per split (whole 32-token tiles)
  int32_t nsplit_comp;    // splits over compressed tokens, per unit
  int32_t nsplit;         // + 1 if the buffer is non-empty
  int32_t total_splits;   // units * nsplit: one warp each
  int32_t warp_bytes;     // shared memory per warp
  TileLayout tl;
};

struct DenseArgs {
  CacheView C;
  int32_t dtype;
  int32_t U, bits, g, G, W, k, r_max, n_max, nblk_max, n_b;
  int32_t n_comp, n_buf, blk0_len, blk0_rank, buffer_rank;
  float* out;             // [U][n_comp + n_buf][128]
};

void decode_plan(DecodeArgs& a, int num_sms);
size_t decode_workspace_bytes(int B, int Hq, int nsplit);
cudaError_t decode_launch(const DecodeArgs& a, cudaStream_t st);
cudaError_t dense_launch(const DenseArgs& a, cudaStream_t st);

}  // namespace gear
