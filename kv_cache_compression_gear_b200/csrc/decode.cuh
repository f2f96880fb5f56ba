// decode.cuh -- argument blocks of the GEAR decode-attention kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gear {

constexpr int kDTile = 32;       // tokens per decode tile (one per lane)
// token stride of one group's value weights in shared memory: the two tokens
// and G groups a value-loop step reads fall in distinct banks
constexpr int kWStride = kDTile + 2;
constexpr int kMaxR = 16;        // largest rank

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

// Shared memory of a decode_warp CTA (4 warps), from a 1024-byte-aligned base:
// first the code tiles of all warps (warp w, tile idx at (4w + idx) * cb), then
// one region of `bytes` per warp holding its meta tiles (meta0 + idx * mb), its
// rest tiles (oidx | oval | lf at rest0 + idx * rb), the float scratch and the
// two stage barriers. Tile idx = 2 * stage + tensor (0 = keys, 1 = values).
struct TileLayout {
  int32_t cb, mb, rb;      // bytes per tile: codes, meta, rest
  int32_t oval, lf;        // offsets of oval and lf inside the rest
  int32_t meta0, rest0;    // offsets of tile 0's meta and rest in the warp's region
  int32_t floats;          // offset of the float scratch
  int32_t bars;            // offset of the two stage barriers
  int32_t bytes;           // bytes of the warp's region, a multiple of 256
  int32_t tx_full;         // bytes a stage barrier expects for a whole, aligned tile
  int32_t tx_part;         // ... for another tile (codes and meta only; the rest is copied by the lanes)
};

// Tensor maps of the codes and meta arrays of both tensors ([U * n_max] rows).
// The meta maps are used when G >= 2 (a meta row of one group is 8 bytes,
// below the 16-byte minimum of a tensor copy).
struct DecodeMaps {
  CUtensorMap kc, vc, km, vm;
};

struct DecodeArgs {
  CacheView K, V;
  int32_t dtype;          // cache dtype
  int32_t B, H, Hq, hq;   // hq = Hq / H query heads per kv head
  int32_t bits, g, G, W, k, r_max;
  int32_t meta_f16;       // (scale, zero) pairs stored as binary16
  int32_t kc, ch_slots;   // K quantized per channel over token groups; token-group slots per unit
  int32_t n_max, nblk_max, n_b;
  int32_t n_comp, n_buf;
  int32_t blk0_len, blk0_rank, buffer_rank;
  float scale_log2;       // softmax scale * log2(e)
  uint32_t one_bits;      // 0x3F800000 (1.0f), passed so that it stays in a register
  const void* q;          // [B][Hq][128] cache dtype
  void* out;              // [B][Hq][128] out dtype
  int32_t out_dtype;
  float* part;            // [B][Hq][nsplit][130] partial (m, l, acc[128]) per warp that meets the unit
  const int32_t* plen;    // [B] device: real tokens at the head of block 0 per batch row, or null (all)
  // paged layout (null table: contiguous). Token t of row b, head h is row
  // (table[b * ppr + t / page_tokens] * H + h) * page_tokens + t % page_tokens
  // of the per-token arrays; rows [3][B] holds each row's block-0 length,
  // blocks and buffer fill (n_comp and n_buf above are the maxima over rows).
  const int32_t* table;
  const int32_t* rows;
  int32_t page_tokens, ppr, num_pages;
  int64_t tot_tokens;     // paged layout: compressed tokens of all units (H * sum of the rows' lengths)
  int32_t seg_tokens;     // compressed tokens per warp (a multiple of 32); 0 without any
  int32_t nsplit;         // partial rows per unit: at most ceil(n_comp / seg_tokens) + 1 warps meet a unit
  int32_t total_splits;   // warps: ceil(units * n_comp / seg_tokens), or units without compressed tokens
  TileLayout tl;
};

struct DenseArgs {
  CacheView C;
  int32_t dtype;
  int32_t U, bits, g, G, W, k, r_max, n_max, nblk_max, n_b;
  int32_t meta_f16;
  int32_t ch, ch_slots;   // per-channel key groups: meta per token-group slot
  int32_t n_comp, n_buf, blk0_len, blk0_rank, buffer_rank;
  float* out;             // [U][n_comp + n_buf][128]
};

void decode_plan(DecodeArgs& a, int num_sms);
// decode_warp launches for each cache dtype (decode_f16.cu, decode_bf16.cu, decode_f32.cu)
cudaError_t decode_warp_launch_f16(const DecodeMaps& maps, const DecodeArgs& a, cudaStream_t st);
cudaError_t decode_warp_launch_bf16(const DecodeMaps& maps, const DecodeArgs& a, cudaStream_t st);
cudaError_t decode_warp_launch_f32(const DecodeMaps& maps, const DecodeArgs& a, cudaStream_t st);
// K caches with per-channel key groups, fp16 or bf16 (decode_kc.cu)
cudaError_t decode_warp_launch_kc(const DecodeMaps& maps, const DecodeArgs& a, cudaStream_t st);
size_t decode_workspace_bytes(int B, int Hq, int nsplit);
cudaError_t decode_launch(const DecodeArgs& a, cudaStream_t st);
cudaError_t dense_launch(const DenseArgs& a, cudaStream_t st);

}  // namespace gear
