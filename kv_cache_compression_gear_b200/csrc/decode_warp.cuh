// decode_warp.cuh -- the decode-step attention kernel over a GEAR-compressed KV
// cache and its launch templates, instantiated per cache dtype by
// decode_f16.cu, decode_bf16.cu and decode_f32.cu (compiled in parallel).
//
// One query token per sequence attends to the n_comp compressed tokens and
// the n_buf full-precision buffer tokens of its kv head (GEAR: Efficient KV
// Cache Compression for LLM Inference, Q3, streaming strategy; the compressed
// entries are consumed as D + L Rf^T with the sparse outliers restored).
// The reconstruction is never materialized: for a key token t of block b
//   q . Khat_t = sum_g [ scale_tg * (sum_{c in g} code_tc q_c) + zero_tg * sum_{c in g} q_c ]
//              + L_t . (Rf_b^T q)
//              + sum_{outliers o} q_{c_o} (x_o - zero_{t,g(c_o)} - L_t . Rf_b[c_o])
// and the value side accumulates p_t * (scale*code + zero) per channel, the
// block's low-rank part as (sum_t p_t L_t) Rf_b^T, and the outlier fix-ups.
//
// Split-K (flash-decoding style), stream-K scheduled: the grid is one wave of
// resident warps, and warp w takes compressed tokens [w*T, (w+1)*T) of all
// (batch, kv head) units laid end to end, for all query heads sharing the kv
// head. A unit boundary inside that run starts a new segment with its own
// partial result; the warp that ends a unit also folds in the unit's buffer.
// The warp brings the tiles of both tensors into its own shared memory with
// tensor copies (codes and meta, 16-byte-chunk swizzled so that both the
// per-token and the per-channel reads are free of bank conflicts) and bulk
// copies (outlier channels and values, L rows), double-buffered on two
// mbarriers. It scores with one lane per token straight from the packed
// codes, keeps an online softmax whose reference moves only when the running
// maximum passes it by 2^8, and accumulates values with one lane per 8
// channels and token parity. The value outlier fix-ups are scattered with
// fire-and-forget float reductions into the segment's partial-result row in
// global memory. decode_combine merges a unit's segments by log-sum-exp.
// Caches without outliers (s = 0, the pages' GEAR-L variant: quantization plus
// low rank) run an instantiation with the outlier code compiled out
// (OUT = false).
#pragma once

#include <string.h>
#include "common.cuh"
#include "decode.cuh"

namespace gear {

constexpr int kDThreads = 128;   // 4 warps, each an independent split
constexpr float kLazy = 8.0f;    // log2 slack of the softmax reference

template <typename T>
__device__ __forceinline__ float load_elem(const void* p, size_t i) {
  if constexpr (sizeof(T) == 4) return reinterpret_cast<const float*>(p)[i];
  else if constexpr (std::is_same<T, __half>::value) return __half2float(reinterpret_cast<const __half*>(p)[i]);
  else return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
}

template <typename T>
__device__ __forceinline__ float load_lfac(const void* p, size_t i) {
  if constexpr (sizeof(T) == 4) return reinterpret_cast<const float*>(p)[i];
  else return __half2float(reinterpret_cast<const __half*>(p)[i]);
}

__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// blocks of a unit whose block 0 holds b0 tokens
__device__ __forceinline__ int block_of(const DecodeArgs& a, int b0, int t) {
  return t < b0 ? 0 : 1 + (t - b0) / a.n_b;
}
__device__ __forceinline__ int block_end(const DecodeArgs& a, int b0, int b) {
  return b == 0 ? b0 : b0 + b * a.n_b;
}

// Bulk copy global -> shared, completing on an mbarrier (no multicast).
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// 2-D tensor copy global -> shared at column 0, row y (no multicast).
__device__ __forceinline__ void tensor_copy(uint32_t dst, const CUtensorMap* map, uint32_t bar, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(0), "r"(y)
      : "memory");
}

// Accesses of the split's partial-result row that go to the L2 point of
// coherence, where the value outlier reductions land.
__device__ __forceinline__ void red_add_gpu(float* p, float v) {
  asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}
__device__ __forceinline__ float ld_gpu(const float* p) {
  float v;
  asm volatile("ld.relaxed.gpu.global.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_gpu(float* p, float v) {
  asm volatile("st.relaxed.gpu.global.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// The 16-byte-chunk swizzle a tensor copy applies to a tile of R-byte rows
// (R = 32, 64, 128: the 32-, 64- and 128-byte modes): byte o of row t lands at
// t*R + (o ^ (swz(t) << 4)), swz(t) = ((t*R) >> 7) & (R/16 - 1). It repeats
// every 8 rows.
template <int R>
__device__ __forceinline__ int swz(int t) {
  return ((t * R) >> 7) & (R / 16 - 1);
}

template <typename T>
__device__ __forceinline__ float l_at(const uint8_t* lf, int t, int j, int rm) {
  if constexpr (sizeof(T) == 4) return reinterpret_cast<const float*>(lf)[t * rm + j];
  else return __half2float(reinterpret_cast<const __half*>(lf)[t * rm + j]);
}

__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
// register-pair moves (no integer arithmetic) for the f32x2 operands
__device__ __forceinline__ uint64_t pk2(float x, float y) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(x), "f"(y));
  return r;
}
__device__ __forceinline__ float lo2(uint64_t v) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
  return a;
}
__device__ __forceinline__ float hi2(uint64_t v) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
  return b;
}

// One token's meta row in shared memory. With binary32 metadata (MF false),
// (scale, zero) of group gi sits at byte (8*gi) ^ mx of the row, mx the lane's
// swizzle term (0 unless G = 4, the only 32-byte row); with binary16 metadata
// the pair is a half2 at byte 4*gi of a row of at most 16 bytes (no swizzle).
template <bool MF>
__device__ __forceinline__ float2 meta_at(const uint8_t* mrow, int gi, int mx) {
  if constexpr (MF) return __half22float2(*reinterpret_cast<const __half2*>(mrow + 4 * gi));
  else return *reinterpret_cast<const float2*>(mrow + ((gi << 3) ^ mx));
}
// The whole row, read in pieces of up to 16 bytes (conflict-free across the lanes).
template <bool MF>
__device__ __forceinline__ void meta_row(const uint8_t* mrow, int G, int mx, float2 (&sz)[4]) {
  if constexpr (MF) {
    if (G == 4) {
      const uint4 a = *reinterpret_cast<const uint4*>(mrow);
      sz[0] = __half22float2(*reinterpret_cast<const __half2*>(&a.x));
      sz[1] = __half22float2(*reinterpret_cast<const __half2*>(&a.y));
      sz[2] = __half22float2(*reinterpret_cast<const __half2*>(&a.z));
      sz[3] = __half22float2(*reinterpret_cast<const __half2*>(&a.w));
    } else if (G == 2) {
      const uint2 a = *reinterpret_cast<const uint2*>(mrow);
      sz[0] = __half22float2(*reinterpret_cast<const __half2*>(&a.x));
      sz[1] = __half22float2(*reinterpret_cast<const __half2*>(&a.y));
      sz[2] = sz[3] = make_float2(0.0f, 0.0f);
    } else {
      sz[0] = __half22float2(*reinterpret_cast<const __half2*>(mrow));
      sz[1] = sz[2] = sz[3] = make_float2(0.0f, 0.0f);
    }
    return;
  }
  if (G == 4) {
    const float4 a = *reinterpret_cast<const float4*>(mrow + mx);
    const float4 b = *reinterpret_cast<const float4*>(mrow + (16 ^ mx));
    sz[0] = make_float2(a.x, a.y); sz[1] = make_float2(a.z, a.w);
    sz[2] = make_float2(b.x, b.y); sz[3] = make_float2(b.z, b.w);
  } else if (G == 2) {
    const float4 a = *reinterpret_cast<const float4*>(mrow);
    sz[0] = make_float2(a.x, a.y); sz[1] = make_float2(a.z, a.w);
    sz[2] = sz[3] = make_float2(0.0f, 0.0f);
  } else {
    sz[0] = *reinterpret_cast<const float2*>(mrow);
    sz[1] = sz[2] = sz[3] = make_float2(0.0f, 0.0f);
  }
}

// Outlier fix-ups of one token: for up to kFast outliers, the channel and the
// difference between the exact value and what codes + low rank give there:
// fix = x_o - (zero_g(c_o) + L_t . Rf[c_o]). Rf rows are 16-byte vectors, so a
// rank <= 4 block needs one load per outlier. All loads are issued together.
// Three slots cover s <= 2 % of 128 channels; more outliers take the general loop.
constexpr int kFast = 3;
template <typename T, bool MF, bool ZC = false, int NS = kFast, int NR = 4>
__device__ __forceinline__ void outlier_fixes(const uint8_t* rest, int oval_off, const uint8_t* mrow, int mx, int t,
                                              int k, int lg, const float (&lt)[NR], const float* rf, int rp,
                                              int (&cix)[NS], float (&fix)[NS], const float* zc = nullptr,
                                              int i0 = 0) {
  float xo[NS], zr[NS];
  float4 rv[NS][NR / 4];
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    const bool on = i0 + i < k;
    cix[i] = on ? rest[t * k + i0 + i] : 0;
    xo[i] = on ? (float)reinterpret_cast<const T*>(rest + oval_off)[t * k + i0 + i] : 0.0f;
  }
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    const bool on = i0 + i < k;
    // the zero point at the outlier's channel: per channel (ZC) or of its group
    zr[i] = on ? (ZC ? zc[cix[i]] : meta_at<MF>(mrow, cix[i] >> lg, mx).y) : 0.0f;
    // only the row's own rp floats: past them lies the next channel's row, or
    // for channel 127 the next block's, which may never have been written (the
    // first float4 is always inside the row, rp >= 4)
#pragma unroll
    for (int q = 0; q < NR / 4; ++q)
      rv[i][q] = (on && (q == 0 || 4 * q < rp)) ? __ldg(reinterpret_cast<const float4*>(rf + cix[i] * rp) + q)
                                               : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  }
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    float lr = 0.0f;
#pragma unroll
    for (int q = 0; q < NR / 4; ++q) {
      lr = fmaf(lt[4 * q], rv[i][q].x, lr);
      lr = fmaf(lt[4 * q + 1], rv[i][q].y, lr);
      lr = fmaf(lt[4 * q + 2], rv[i][q].z, lr);
      lr = fmaf(lt[4 * q + 3], rv[i][q].w, lr);
    }
    fix[i] = i0 + i < k ? xo[i] - (zr[i] + lr) : 0.0f;
  }
}

// Low-rank value at channel c for any rank: L_t . Rf[c] over rb <= 16 ranks.
template <typename T>
__device__ __forceinline__ float lowrank_at(const uint8_t* lf, int t, int rm, int rb, const float* rf, int rp, int c) {
  float lr = 0.0f;
  for (int j4 = 0; j4 < rb; j4 += 4) {
    const float4 r4 = __ldg(reinterpret_cast<const float4*>(rf + c * rp + j4));
    const float rr[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
      if (j4 + jj < rb) lr = fmaf(l_at<T>(lf, t, j4 + jj, rm), rr[jj], lr);
  }
  return lr;
}

// Shared memory (see TileLayout): the warps' code tiles, then per warp 4 meta
// tiles | 4 rest tiles | floats | 2 mbarriers. Floats: qw [HQ][128] (q scaled
// by the code weights; q itself is qw * CF::weight, exactly) | u [HQ][16] |
// alr [HQ][16] | w [32][G][HQ] | accx [HQ][128] and, for keys quantized per
// channel over token groups (KC, the KIVI-combined cache), qk [HQ][128] (qw
// times the channel's scale in the current key group) | zk [128] (the group's
// per-channel zero points). The [HQ][128] arrays hold channel c at slot c;
// loops that touch all of them use slot e*32 + lane so that every lane stays in
// its own bank.
template <typename T, int BITS, int HQ, bool OUT, bool MF, bool KC>
__global__ void __launch_bounds__(kDThreads, HQ <= 2 ? 4 : (HQ == 4 ? 2 : 1)) decode_warp(const __grid_constant__ DecodeMaps maps,
                                                         const DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t dsm[];
  constexpr int W = 4 * BITS;
  constexpr int R = 4 * W;   // code bytes per token
  constexpr int kRReg = 4;   // value low-rank weights kept in registers
  using CF = CodeFloats<BITS>;
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gs = blockIdx.x * 4 + wid;
  if (gs >= a.total_splits) return;
  const TileLayout& L = a.tl;
  const int G = a.G, rm = a.r_max, k = a.k;
  const int rp = rpad_of(rm);
  const uint32_t one = a.one_bits;
  const int lg = a.g == 32 ? 5 : (a.g == 64 ? 6 : 7);
  uint8_t* cta = align_smem_1024(dsm);
  uint8_t* cb = cta + (size_t)wid * 4 * L.cb;                          // this warp's 4 code tiles
  uint8_t* wb = cta + (size_t)16 * L.cb + (size_t)wid * L.bytes;     // its other regions
  float* qw_s = reinterpret_cast<float*>(wb + L.floats);
  float* u_s = qw_s + HQ * 128;
  float* alr_s = u_s + HQ * kMaxR;   // value low-rank weights j >= kRReg
  float* w_s = alr_s + HQ * kMaxR;
  float* accx_s = w_s + kWStride * G * HQ;
  float* qk_s = accx_s + HQ * 128;   // KC only
  float* zk_s = qk_s + HQ * 128;     // KC only
  uint64_t* bars = reinterpret_cast<uint64_t*>(wb + L.bars);

  // value side: lane owns channels 8*(lane & 15) .. +7 and tokens of parity lane >> 4
  const int lq = lane & 15, par = lane >> 4;
  const int my_g = (8 * lq) >> lg;
  if (lane == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbarrier_init();
  }
  __syncwarp();
  int it = 0;   // tiles staged so far; the stage parities run on across segments

  // One segment: compressed tokens [c0, c1) of `unit` (maybe none), then the
  // unit's buffer if with_buf, into partial row sp of the unit. Returns false if
  // a bounded wait gave up (the error word is set; nothing is written).
  auto segment = [&](const int unit, const int c0, const int c1_run, const int sp, const bool with_buf) -> bool {
    const int b = unit / a.H, h = unit % a.H;
    // this row's block-0 length, compressed tokens and buffer fill (paged
    // layout: per row, the run cut to the row's own tokens)
    int b0 = a.blk0_len, nbuf = a.n_buf, c1 = c1_run;
    if (a.rows) {
      b0 = __ldg(a.rows + b);
      const int nblk = __ldg(a.rows + a.B + b);
      nbuf = __ldg(a.rows + 2 * a.B + b);
      c1 = max(c0, min(c1_run, nblk > 0 ? b0 + (nblk - 1) * a.n_b : 0));
    }
    const bool comp = c1 > c0;
    // right-padded prefill: block-0 tokens [pl, b0) of this batch row are
    // padding and take no part in the softmax
    const int pl = a.plen ? min(max(__ldg(a.plen + b), 0), b0) : b0;
    // this split's partial row of query head hh: part_row + hh * hstride
    float* part_row = a.part + (((size_t)b * a.Hq + (size_t)h * HQ) * a.nsplit + sp) * 130;
    const size_t hstride = (size_t)a.nsplit * 130;
    for (int e = lane; e < HQ * 128; e += 32) {
      const float qv = load_elem<T>(a.q, ((size_t)b * a.Hq + (size_t)h * HQ + (e >> 7)) * 128 + (e & 127));
      qw_s[e] = qv * CF::inv_weight(e & 127);
      accx_s[e] = 0.0f;
      if (OUT && comp) st_gpu(part_row + (e >> 7) * hstride + 2 + (e & 127), 0.0f);   // value outlier sums
    }
    for (int e = lane; e < HQ * kMaxR; e += 32) alr_s[e] = 0.0f;
    __syncwarp();

    float m[HQ], lsum[HQ], sw[HQ][4], spm[HQ][4], alr[HQ][kRReg];
    uint64_t acc[HQ][4];   // channel pairs (8 channels)
#pragma unroll
    for (int hh = 0; hh < HQ; ++hh) {
      m[hh] = -INFINITY;
      lsum[hh] = 0.0f;
#pragma unroll
      for (int e = 0; e < 4; ++e) { acc[hh][e] = 0; sw[hh][e] = 0.0f; spm[hh][e] = 0.0f; alr[hh][e] = 0.0f; }
    }

    int rb = 0;   // rank of the current block

    // Moves the softmax reference of head hh to mt if mt passes it by more than
    // 2^kLazy, rescaling every accumulator (registers, shared memory and the
    // value outlier sums in global memory).
    auto move_ref = [&](const int hh, const float mt) {
      if (mt > m[hh] + kLazy) {   // warp-uniform
        if (m[hh] != -INFINITY) {
          const float al = exp2f(m[hh] - mt);
          lsum[hh] *= al;
          const uint64_t al2 = pk2(al, al);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[hh][e] = fma2(acc[hh][e], al2, 0);
            sw[hh][e] *= al;
            spm[hh][e] *= al;
            alr[hh][e] *= al;
            accx_s[hh * 128 + e * 32 + lane] *= al;
          }
          if (rb > kRReg && lane < kMaxR) alr_s[hh * kMaxR + lane] *= al;
          if constexpr (OUT) {
            if (comp) {
              __threadfence();
              __syncwarp();
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float* pc = part_row + hh * hstride + 2 + e * 32 + lane;
                st_gpu(pc, ld_gpu(pc) * al);
              }
              __threadfence();
              __syncwarp();
            }
          }
        }
        m[hh] = mt;
      }
    };

    if (comp) {
      __threadfence();   // the zeroed outlier sums before any reduction
      __syncwarp();

      // group sums of q and of the weighted q, per 32-channel block
      float qs_blk[HQ][4], qw_blk[HQ][4];
#pragma unroll
      for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
        for (int bk = 0; bk < 4; ++bk) {
          qs_blk[hh][bk] = warp_sum(qw_s[hh * 128 + bk * 32 + lane] * CF::weight(bk * 32 + lane));
          qw_blk[hh][bk] = warp_sum(qw_s[hh * 128 + bk * 32 + lane]);
        }

      // ---- copy roles: lanes 0/1 codes (K/V), 2/3 meta by tensor copy (G >= 2),
      // 4/5 oidx, 6/7 oval, 8/9 L rows, 10/11 meta by bulk copy (rows under 16 bytes)
      const int mrb = MF ? 4 * G : 8 * G;   // meta bytes per token
      const bool meta_tma = mrb >= 16;
      const int x = lane & 1;
      const CUtensorMap* my_map = nullptr;
      const uint8_t* my_src = nullptr;
      int my_bpr = 0;
      uint32_t my_dst = 0, my_sst = 0;
      {
        const int esz = (int)sizeof(T), lsz = sizeof(T) == 4 ? 4 : 2;
        const uint32_t wbs = smem_u32(wb);
        switch (lane >> 1) {
          case 0:
            my_map = x ? &maps.vc : &maps.kc;
            my_dst = smem_u32(cb) + x * L.cb;
            my_sst = 2 * L.cb;
            break;
          case 1:
            if (meta_tma && !(KC && x == 0)) {   // per-channel key groups have no per-token meta rows
              my_map = x ? &maps.vm : &maps.km;
              my_dst = wbs + L.meta0 + x * L.mb;
              my_sst = 2 * L.mb;
            }
            break;
          case 2:
            my_src = x ? a.V.oidx : a.K.oidx;
            my_bpr = k;
            my_dst = wbs + L.rest0 + x * L.rb;
            my_sst = 2 * L.rb;
            break;
          case 3:
            my_src = reinterpret_cast<const uint8_t*>(x ? a.V.oval : a.K.oval);
            my_bpr = k * esz;
            my_dst = wbs + L.rest0 + x * L.rb + L.oval;
            my_sst = 2 * L.rb;
            break;
          case 4:
            my_src = reinterpret_cast<const uint8_t*>(x ? a.V.lfac : a.K.lfac);
            my_bpr = rm * lsz;
            my_dst = wbs + L.rest0 + x * L.rb + L.lf;
            my_sst = 2 * L.rb;
            break;
          case 5:
            if (!meta_tma && !(KC && x == 0)) {
              my_src = reinterpret_cast<const uint8_t*>(x ? a.V.meta : a.K.meta);
              my_bpr = mrb;
              my_dst = wbs + L.meta0 + x * L.mb;
              my_sst = 2 * L.mb;
            }
            break;
          default:
            break;
        }
      }
      const size_t row0 = (size_t)unit * a.n_max;   // row of the unit's token 0 (contiguous layout)
      // paged layout: the row of token t (a 32-token tile never spans two pages)
      auto token_row = [&](int t) -> size_t {
        if (!a.table) return row0 + t;
        const int pg = min(max(__ldg(a.table + (size_t)b * a.ppr + t / a.page_tokens), 0), a.num_pages - 1);
        return ((size_t)pg * a.H + h) * a.page_tokens + t % a.page_tokens;
      };
      // Brings tokens [t, t + nt) of the unit into stage s. A whole, 32-aligned
      // tile is all copies; another one (a block boundary or the split's end)
      // takes codes and meta by tensor copy (rows past nt are read and ignored)
      // and the rest by plain loads of the lanes.
      auto issue = [&](int s, int t, int nt) {
        const bool full = nt == kDTile && (t & (kDTile - 1)) == 0;
        if (lane == 0) mbar_arrive_expect_tx(&bars[s], (uint32_t)(full ? L.tx_full : L.tx_part));
        __syncwarp();
        const uint32_t bar = smem_u32(&bars[s]);
        const size_t row = token_row(t);
        if (my_map) {
          fence_proxy_async_smem();
          tensor_copy(my_dst + s * my_sst, my_map, bar, (int32_t)row);
        } else if (full && my_bpr > 0) {
          fence_proxy_async_smem();
          bulk_copy(my_dst + s * my_sst, my_src + row * my_bpr, (uint32_t)(kDTile * my_bpr), bar);
        }
        if (!full) {
          const int esz = (int)sizeof(T), lsz = sizeof(T) == 4 ? 4 : 2;
#pragma unroll
          for (int xx = 0; xx < 2; ++xx) {
            const CacheView& cv = xx ? a.V : a.K;
            uint8_t* rest = wb + L.rest0 + (2 * s + xx) * L.rb;
            const uint8_t* oi = cv.oidx + row * k;
            for (int e = lane; e < nt * k; e += 32) rest[e] = oi[e];
            const uint8_t* ov = reinterpret_cast<const uint8_t*>(cv.oval) + row * k * esz;
            for (int e = lane; e < nt * k * esz; e += 32) rest[L.oval + e] = ov[e];
            const uint8_t* lf = reinterpret_cast<const uint8_t*>(cv.lfac) + row * rm * lsz;
            for (int e = lane; e < nt * rm * lsz; e += 32) rest[L.lf + e] = lf[e];
            if (!meta_tma && !(KC && xx == 0)) {
              uint8_t* md = wb + L.meta0 + (2 * s + xx) * L.mb;
              const uint8_t* ms = reinterpret_cast<const uint8_t*>(cv.meta) + row * mrb;
              for (int e = lane; e < nt * mrb; e += 32) md[e] = ms[e];
            }
          }
        }
      };

      // blocks: block 0 = [0, blk0_len), then n_b tokens each; tracked incrementally
      int blk = block_of(a, b0, c0);
      int bend = block_end(a, b0, blk);
      const float* rfk = nullptr;
      const float* rfv = nullptr;
      // KC: slot and end of the key token group holding token t of block b
      // (block 0 in groups of g from 0; a flushed block holds whole groups)
      auto kgroup = [&](int t, int b, int& slot, int& gend) {
        if (b == 0) {
          const int j = t / a.g;
          slot = j;
          gend = min((j + 1) * a.g, b0);
        } else {
          const int bs = block_end(a, b0, b - 1), j = (t - bs) / a.g;
          slot = (b0 + a.g - 1) / a.g + (b - 1) * (a.n_b / a.g) + j;
          gend = bs + (j + 1) * a.g;
        }
      };
      // tiles follow the unit's 32-token grid: [t, next multiple of 32), clipped
      // to the split, the block and (KC) the key group
      auto next_end = [&](int t, int be, int b) {
        int e = min(min((t & ~(kDTile - 1)) + kDTile, c1), be);
        if constexpr (KC) {
          int sl, ge;
          kgroup(t, b, sl, ge);
          e = min(e, ge);
        }
        return e;
      };
      issue(it & 1, c0, next_end(c0, bend, blk) - c0);
      int kslot = -1;       // KC: key group whose qk, zk are loaded
      float ksub[HQ], kz[HQ];   // KC: sum of qk, and q . zero over the group's channels
#pragma unroll
      for (int hh = 0; hh < HQ; ++hh) { ksub[hh] = 0.0f; kz[hh] = 0.0f; }

      // lane-constant swizzle terms: key rows (lane = token), meta rows, and the
      // value reads of token 2*i + par (period 4 in i)
      const int xs = swz<R>(lane);
      const int mx = mrb == 32 ? ((lane >> 2) & 1) << 4 : 0;
      int voff[4];
      {
        const int ob = BITS == 4 ? 4 * lq : (BITS == 2 ? 2 * lq : 8 * lq);
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) voff[mm] = ob ^ (swz<R>(2 * mm + par) << 4);
      }

      // finishes the value low-rank part of the current block: accx += alr Rf_v^T
      auto finish_block = [&]() {
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
          for (int j = 0; j < kRReg; ++j) alr[hh][j] = warp_sum(alr[hh][j]);
        __syncwarp();
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = e * 32 + lane;
            float v = accx_s[hh * 128 + c];
            const float4 r0 = __ldg(reinterpret_cast<const float4*>(rfv + c * rp));
            v = fmaf(alr[hh][0], r0.x, v);
            v = fmaf(alr[hh][1], r0.y, v);
            v = fmaf(alr[hh][2], r0.z, v);
            v = fmaf(alr[hh][3], r0.w, v);
            for (int j4 = kRReg; j4 < rb; j4 += 4) {
              const float4 r4 = __ldg(reinterpret_cast<const float4*>(rfv + c * rp + j4));
              v = fmaf(alr_s[hh * kMaxR + j4], r4.x, v);
              v = fmaf(alr_s[hh * kMaxR + j4 + 1], r4.y, v);
              v = fmaf(alr_s[hh * kMaxR + j4 + 2], r4.z, v);
              v = fmaf(alr_s[hh * kMaxR + j4 + 3], r4.w, v);
            }
            accx_s[hh * 128 + c] = v;
          }
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
          for (int j = 0; j < kRReg; ++j) alr[hh][j] = 0.0f;
        __syncwarp();
        for (int e = lane; e < HQ * kMaxR; e += 32) alr_s[e] = 0.0f;
      };

      int t0 = c0, cur_blk = -1;
      while (t0 < c1) {
        if (t0 >= bend) { ++blk; bend = block_end(a, b0, blk); }
        const int t1 = next_end(t0, bend, blk);
        const int nt = t1 - t0;
        const int s = it & 1;
        if (t1 < c1) {   // prefetch the next tile into the other stage
          const int b2 = t1 >= bend ? blk + 1 : blk;
          issue(s ^ 1, t1, next_end(t1, block_end(a, b0, b2), b2) - t1);
        }
        const bool landed = mbar_wait(&bars[s], (uint32_t)(it >> 1) & 1u);
        if (!__all_sync(0xFFFFFFFFu, landed)) {
          // give up on this split; let the other stage's copies land first
          if (t1 < c1) mbar_wait(&bars[s ^ 1], (uint32_t)((it + 1) >> 1) & 1u);
          return false;
        }
        __syncwarp();
        const uint8_t* tkc = cb + (2 * s) * L.cb;
        const uint8_t* tvc = tkc + L.cb;
        const uint8_t* tkm = wb + L.meta0 + (2 * s) * L.mb;
        const uint8_t* tvm = tkm + L.mb;
        const uint8_t* tkr = wb + L.rest0 + (2 * s) * L.rb;
        const uint8_t* tvr = tkr + L.rb;

        if (blk != cur_blk) {
          // finish the previous block's value low-rank part, then switch Rf
          if (cur_blk >= 0) finish_block();
          cur_blk = blk;
          rb = blk == 0 ? a.blk0_rank : a.buffer_rank;
          const size_t rf0 = ((size_t)unit * a.nblk_max + blk) * 128 * rp;
          rfk = a.K.rfac + rf0;
          rfv = a.V.rfac + rf0;
          // u = Rf_k^T q for every query head
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh)
            for (int j4 = 0; j4 < rb; j4 += 4) {
              float u4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c = e * 32 + lane;
                const float4 r4 = __ldg(reinterpret_cast<const float4*>(rfk + c * rp + j4));
                const float qv = qw_s[hh * 128 + c] * CF::weight(c);
                u4[0] = fmaf(r4.x, qv, u4[0]);
                u4[1] = fmaf(r4.y, qv, u4[1]);
                u4[2] = fmaf(r4.z, qv, u4[2]);
                u4[3] = fmaf(r4.w, qv, u4[3]);
              }
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) {
                const float v = warp_sum(u4[jj]);
                if (lane == 0) u_s[hh * kMaxR + j4 + jj] = v;
              }
            }
          __syncwarp();
        }

        if constexpr (KC) {
          int sl, ge;
          kgroup(t0, blk, sl, ge);
          if (sl != kslot) {   // a new key group: its per-channel scales and zero points
            kslot = sl;
            const float2* km = reinterpret_cast<const float2*>(a.K.meta) + ((size_t)unit * a.ch_slots + sl) * 128;
            float ps[HQ], pz[HQ];
#pragma unroll
            for (int hh = 0; hh < HQ; ++hh) { ps[hh] = 0.0f; pz[hh] = 0.0f; }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = e * 32 + lane;
              const float2 sz = __ldg(km + c);
              zk_s[c] = sz.y;
#pragma unroll
              for (int hh = 0; hh < HQ; ++hh) {
                const float qw = qw_s[hh * 128 + c];
                const float qk = qw * sz.x;
                qk_s[hh * 128 + c] = qk;
                ps[hh] += qk;
                pz[hh] = fmaf(qw * CF::weight(c), sz.y, pz[hh]);
              }
            }
#pragma unroll
            for (int hh = 0; hh < HQ; ++hh) { ksub[hh] = warp_sum(ps[hh]); kz[hh] = warp_sum(pz[hh]); }
            __syncwarp();
          }
        }

        // ---------------- scores: lane = token
        const int t = lane;
        const bool live = t < nt && (t0 + t < pl || t0 + t >= b0);
        const uint8_t* kmrow = tkm + t * mrb;
        const uint8_t* vmrow = tvm + t * mrb;
        float s_[HQ];
        {
          const uint8_t* crow = tkc + t * R;
          // per 32-channel block: four independent f32x2 chains while the block's
          // 16 bytes are read (one block per 16-byte load for 4-bit codes, then
          // summed into fb), or two chains per block kept to the end otherwise
          constexpr bool kOneBlk = CF::kPerWord * 4 == 32;
          uint64_t sb[HQ][4][2];
          float fb[HQ][4];
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
            for (int bk = 0; bk < 4; ++bk) { sb[hh][bk][0] = 0; sb[hh][bk][1] = 0; fb[hh][bk] = 0.0f; }
#pragma unroll
          for (int j = 0; j < W / 4; ++j) {
            const uint4 wv = *reinterpret_cast<const uint4*>(crow + ((j ^ xs) << 4));
            const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
            uint64_t c4[HQ][4];
#pragma unroll
            for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
              for (int e = 0; e < 4; ++e) c4[hh][e] = 0;
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
              const int cbase = (4 * j + wi) * CF::kPerWord;
              const int bk = cbase >> 5;
              float f[CF::kPerWord];
              CF::word(wd[wi], f, one);
#pragma unroll
              for (int e = 0; e < CF::kPerWord; e += 4) {
                const int ch = ((cbase + e) >> 2) & 1;
#pragma unroll
                for (int hh = 0; hh < HQ; ++hh) {
                  const float4 qv = *reinterpret_cast<const float4*>((KC ? qk_s : qw_s) + hh * 128 + cbase + e);
                  if constexpr (kOneBlk) {
                    c4[hh][2 * ch] = fma2(pk2(f[e], f[e + 1]), pk2(qv.x, qv.y), c4[hh][2 * ch]);
                    c4[hh][2 * ch + 1] = fma2(pk2(f[e + 2], f[e + 3]), pk2(qv.z, qv.w), c4[hh][2 * ch + 1]);
                  } else {
                    sb[hh][bk][ch] = fma2(pk2(f[e], f[e + 1]), pk2(qv.x, qv.y), sb[hh][bk][ch]);
                    sb[hh][bk][ch] = fma2(pk2(f[e + 2], f[e + 3]), pk2(qv.z, qv.w), sb[hh][bk][ch]);
                  }
                }
              }
            }
            if constexpr (kOneBlk) {
#pragma unroll
              for (int hh = 0; hh < HQ; ++hh)
                fb[hh][j] = ((lo2(c4[hh][0]) + hi2(c4[hh][0])) + (lo2(c4[hh][1]) + hi2(c4[hh][1]))) +
                            ((lo2(c4[hh][2]) + hi2(c4[hh][2])) + (lo2(c4[hh][3]) + hi2(c4[hh][3])));
            }
          }
          if constexpr (!kOneBlk) {
#pragma unroll
            for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
              for (int bk = 0; bk < 4; ++bk)
                fb[hh][bk] = (lo2(sb[hh][bk][0]) + hi2(sb[hh][bk][0])) + (lo2(sb[hh][bk][1]) + hi2(sb[hh][bk][1]));
          }
          float2 sz[4];
          if constexpr (!KC) meta_row<MF>(kmrow, G, mx, sz);
          const int bpg = a.g >> 5;   // 32-channel blocks per group
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh) {
            if constexpr (KC) {   // sum_c scale_c q_c code_c + q . zero of the key group
              s_[hh] = ((fb[hh][0] + fb[hh][1]) + (fb[hh][2] + fb[hh][3])) - ksub[hh] + kz[hh];
              continue;
            }
            float v = 0.0f;
#pragma unroll
            for (int gi = 0; gi < 4; ++gi) {
              if (gi >= G) break;
              float f = 0.0f, qsw = 0.0f, qss = 0.0f;
#pragma unroll
              for (int bk = 0; bk < 4; ++bk)
                if ((bk / bpg) == gi) {
                  f += fb[hh][bk];
                  qsw += qw_blk[hh][bk];
                  qss += qs_blk[hh][bk];
                }
              v = fmaf(sz[gi].x, f - qsw, v);
              v = fmaf(sz[gi].y, qss, v);
            }
            s_[hh] = v;
          }
          if (live) {
            // low-rank part and outlier fix-ups
            float lt[kRReg];
#pragma unroll
            for (int j = 0; j < kRReg; ++j) lt[j] = j < rb ? l_at<T>(tkr + L.lf, t, j, rm) : 0.0f;
#pragma unroll
            for (int j = 0; j < kRReg; ++j)
#pragma unroll
              for (int hh = 0; hh < HQ; ++hh) s_[hh] = fmaf(lt[j], j < rb ? u_s[hh * kMaxR + j] : 0.0f, s_[hh]);
            for (int j = kRReg; j < rb; ++j) {
              const float lj = l_at<T>(tkr + L.lf, t, j, rm);
#pragma unroll
              for (int hh = 0; hh < HQ; ++hh) s_[hh] = fmaf(lj, u_s[hh * kMaxR + j], s_[hh]);
            }
            if constexpr (!OUT) {
            } else if (k <= kFast && rb <= kRReg) {
              int cix[kFast];
              float fx[kFast];
              outlier_fixes<T, MF, KC>(tkr, L.oval, kmrow, mx, t, k, lg, lt, rfk, rp, cix, fx, zk_s);
#pragma unroll
              for (int i = 0; i < kFast; ++i)
#pragma unroll
                for (int hh = 0; hh < HQ; ++hh) s_[hh] = fmaf(qw_s[hh * 128 + cix[i]] * CF::weight(cix[i]), fx[i], s_[hh]);
            } else if (k <= 8 && rb <= 8) {
              // the token's L row once, then outliers four at a time
              float l8[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) l8[j] = j < kRReg ? lt[j] : (j < rb ? l_at<T>(tkr + L.lf, t, j, rm) : 0.0f);
#pragma unroll
              for (int i0 = 0; i0 < 8; i0 += 4) {
                if (i0 >= k) break;
                int cix[4];
                float fx[4];
                outlier_fixes<T, MF, KC, 4, 8>(tkr, L.oval, kmrow, mx, t, k, lg, l8, rfk, rp, cix, fx, zk_s, i0);
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                  for (int hh = 0; hh < HQ; ++hh)
                    s_[hh] = fmaf(qw_s[hh * 128 + cix[i]] * CF::weight(cix[i]), fx[i], s_[hh]);
              }
            } else {
              for (int i = 0; i < k; ++i) {
                const int c = tkr[t * k + i];
                const float lr = lowrank_at<T>(tkr + L.lf, t, rm, rb, rfk, rp, c);
                const float xo = (float)reinterpret_cast<const T*>(tkr + L.oval)[t * k + i];
                const float fix = xo - ((KC ? zk_s[c] : meta_at<MF>(kmrow, c >> lg, mx).y) + lr);
#pragma unroll
                for (int hh = 0; hh < HQ; ++hh) s_[hh] = fmaf(qw_s[hh * 128 + c] * CF::weight(c), fix, s_[hh]);
              }
            }
          }
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh) s_[hh] = live ? s_[hh] * a.scale_log2 : -INFINITY;
        }

        // ---------------- online softmax; the reference m moves only when the
        // tile's maximum passes it by more than 2^kLazy
        float p[HQ];
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh) {
          move_ref(hh, warp_max(s_[hh]));
          p[hh] = live ? exp2f(s_[hh] - m[hh]) : 0.0f;
          lsum[hh] += p[hh];
        }
        // value-side per-token weights w = p * scale; zero-point and low-rank sums
        {
          float2 vsz[4];
          meta_row<MF>(vmrow, G, mx, vsz);
#pragma unroll
          for (int gi = 0; gi < 4; ++gi) {
            if (gi >= G) break;
            const float2 sz = live ? vsz[gi] : make_float2(0.0f, 0.0f);
#pragma unroll
            for (int hh = 0; hh < HQ; ++hh) {
              const float wv = p[hh] * sz.x;
              w_s[(gi * kWStride + t) * HQ + hh] = wv;   // group-major: token stride HQ
              sw[hh][gi] += wv;
              spm[hh][gi] = fmaf(p[hh], sz.y, spm[hh][gi]);
            }
          }
          if (live) {
            float lv[kRReg];
#pragma unroll
            for (int j = 0; j < kRReg; ++j) lv[j] = j < rb ? l_at<T>(tvr + L.lf, t, j, rm) : 0.0f;
#pragma unroll
            for (int j = 0; j < kRReg; ++j)
#pragma unroll
              for (int hh = 0; hh < HQ; ++hh) alr[hh][j] = fmaf(p[hh], lv[j], alr[hh][j]);
            // value outliers: p * fix lands on channel c of the split's row
            if constexpr (!OUT) {
            } else if (k <= kFast && rb <= kRReg) {
              int cix[kFast];
              float fx[kFast];
              outlier_fixes<T, MF>(tvr, L.oval, vmrow, mx, t, k, lg, lv, rfv, rp, cix, fx);
#pragma unroll
              for (int i = 0; i < kFast; ++i)
                if (i < k)
#pragma unroll
                  for (int hh = 0; hh < HQ; ++hh) red_add_gpu(part_row + hh * hstride + 2 + cix[i], p[hh] * fx[i]);
            } else if (k <= 8 && rb <= 8) {
              float l8[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) l8[j] = j < kRReg ? lv[j] : (j < rb ? l_at<T>(tvr + L.lf, t, j, rm) : 0.0f);
#pragma unroll
              for (int i0 = 0; i0 < 8; i0 += 4) {
                if (i0 >= k) break;
                int cix[4];
                float fx[4];
                outlier_fixes<T, MF, false, 4, 8>(tvr, L.oval, vmrow, mx, t, k, lg, l8, rfv, rp, cix, fx, nullptr, i0);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  if (i0 + i < k)
#pragma unroll
                    for (int hh = 0; hh < HQ; ++hh) red_add_gpu(part_row + hh * hstride + 2 + cix[i], p[hh] * fx[i]);
              }
            } else {
              for (int i = 0; i < k; ++i) {
                const int c = tvr[t * k + i];
                const float lr = lowrank_at<T>(tvr + L.lf, t, rm, rb, rfv, rp, c);
                const float xo = (float)reinterpret_cast<const T*>(tvr + L.oval)[t * k + i];
                const float fix = xo - (meta_at<MF>(vmrow, c >> lg, mx).y + lr);
#pragma unroll
                for (int hh = 0; hh < HQ; ++hh) red_add_gpu(part_row + hh * hstride + 2 + c, p[hh] * fix);
              }
            }
          }
        }
        for (int j = kRReg; j < rb; ++j)   // ranks beyond the register slots
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh) {
            const float v = warp_sum(live ? p[hh] * l_at<T>(tvr + L.lf, t, j, rm) : 0.0f);
            if (lane == 0) alr_s[hh * kMaxR + j] += v;
          }
        __syncwarp();

        // ---------------- values: lane = 8 channels, tokens 2*i + par. Tokens
        // past nt have w = 0 (their codes are finite), so every tile runs all 16.
        {
          // per-lane bases advanced by constants; offsets inside a step are
          // compile-time constants. With the outlier code compiled in, the loop
          // stays rolled to keep the kernel inside the instruction cache.
          const uint8_t* vb[4];
#pragma unroll
          for (int mm = 0; mm < 4; ++mm) vb[mm] = tvc + par * R + voff[mm];
          const float* wrow = w_s + (my_g * kWStride + par) * HQ;
#pragma unroll (OUT ? 1 : 4)
          for (int i4 = 0; i4 < kDTile / 2; i4 += 4) {
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) {
              const uint8_t* row = vb[mm] + mm * 2 * R;
              const float* wr = wrow + mm * 2 * HQ;
              float f[8];
              if constexpr (BITS == 4) {
                CF::word(*reinterpret_cast<const uint32_t*>(row), f, one);
              } else if constexpr (BITS == 2) {
                float ff[16];
                CF::word(*reinterpret_cast<const uint16_t*>(row), ff, one);
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = ff[e];
              } else {
                const uint2 ww = *reinterpret_cast<const uint2*>(row);
                float fa[4], fb[4];
                CF::word(ww.x, fa, one);
                CF::word(ww.y, fb, one);
#pragma unroll
                for (int e = 0; e < 4; ++e) { f[e] = fa[e]; f[4 + e] = fb[e]; }
              }
#pragma unroll
              for (int hh = 0; hh < HQ; ++hh) {
                const float wv = wr[hh];
                const uint64_t w2 = pk2(wv, wv);
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[hh][e] = fma2(w2, pk2(f[2 * e], f[2 * e + 1]), acc[hh][e]);
              }
            }
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) vb[mm] += 8 * R;
            wrow += 8 * HQ;
          }
        }
        __syncwarp();
        t0 = t1;
        ++it;
      }
      // last block's value low-rank part
      if (cur_blk >= 0) finish_block();
    }
    if (with_buf) {
      // ---------------- the streaming buffer: exact tokens, lane = token for keys
      const size_t brow = (size_t)unit * a.n_b;
      for (int t0 = 0; t0 < nbuf; t0 += kDTile) {
        const int nt = min(kDTile, nbuf - t0);
        const bool live = lane < nt;
        float s[HQ];
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh) s[hh] = 0.0f;
        if (live) {
          for (int c = 0; c < 128; ++c) {
            const float x = load_elem<T>(a.K.buf, (brow + t0 + lane) * 128 + c);
#pragma unroll
            for (int hh = 0; hh < HQ; ++hh) s[hh] = fmaf(x, qw_s[hh * 128 + c] * CF::weight(c), s[hh]);
          }
        }
        float p[HQ];
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh) {
          const float sv = live ? s[hh] * a.scale_log2 : -INFINITY;
          move_ref(hh, warp_max(sv));
          p[hh] = live ? exp2f(sv - m[hh]) : 0.0f;
          lsum[hh] += p[hh];
        }
        __syncwarp();
        for (int tt = 0; tt < nt; ++tt) {
          float xv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) xv[e] = load_elem<T>(a.V.buf, (brow + t0 + tt) * 128 + e * 32 + lane);
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh) {
            const float pt = __shfl_sync(0xFFFFFFFFu, p[hh], tt);
#pragma unroll
            for (int e = 0; e < 4; ++e) accx_s[hh * 128 + e * 32 + lane] += pt * xv[e];
          }
        }
        __syncwarp();
      }
    }
    if (OUT && comp) __threadfence();   // the value outlier sums, before they are read back
    __syncwarp();

    // ---------------- partial result of this split
#pragma unroll
    for (int hh = 0; hh < HQ; ++hh) {
      const float l_all = warp_sum(lsum[hh]);
      float swg = 0.0f, spg = 0.0f;
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) {
        const float a1 = warp_sum(sw[hh][gi]), a2 = warp_sum(spm[hh][gi]);
        if (gi == my_g) { swg = a1; spg = a2; }
      }
      // the two token parities hold the same channels: add them up
      float v[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = lo2(acc[hh][e]) + __shfl_xor_sync(0xFFFFFFFFu, lo2(acc[hh][e]), 16);
        v[2 * e + 1] = hi2(acc[hh][e]) + __shfl_xor_sync(0xFFFFFFFFu, hi2(acc[hh][e]), 16);
      }
      float* dst = part_row + hh * hstride;
      if (lane == 0) { dst[0] = m[hh]; dst[1] = l_all; }
      if (par == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int c = 8 * lq + e;
          const float corr = (OUT && comp) ? ld_gpu(dst + 2 + c) : 0.0f;
          dst[2 + c] = CF::inv_weight(c) * (v[e] - swg) + spg + accx_s[hh * 128 + c] + corr;
        }
      }
    }
    return true;
  };

  // stream-K: this warp's run [gs * seg_tokens, (gs + 1) * seg_tokens) of the
  // units' compressed tokens, cut at unit boundaries; the warp that ends a unit
  // also takes its buffer. Without compressed tokens, warp gs takes unit gs's
  // buffer.
  // Paged layout: units hold their rows' own lengths, laid end to end row by
  // row (unit b*H + h starts at H * (lengths of rows < b) + h * length of b).
  const int64_t n = a.n_comp;
  const int64_t tot = a.rows ? a.tot_tokens : (int64_t)a.B * a.H * n;
  int64_t gpos = tot > 0 ? (int64_t)gs * a.seg_tokens : 0;
  const int64_t gend = tot > 0 ? min(gpos + (int64_t)a.seg_tokens, tot) : 1;
  while (gpos < gend) {
    int unit, c0, c1, sp;
    bool with_buf;
    if (a.rows && tot > 0) {
      // the row holding position gpos: 32 rows per pass, lane = row, running
      // sums of the rows' token counts (H units each)
      int row = -1, rlen = 0;
      int64_t rstart = 0, base = 0;
      for (int bc = 0; bc < a.B && row < 0; bc += 32) {
        const int bl = bc + lane;
        int len = 0;
        if (bl < a.B) {
          const int nb = __ldg(a.rows + a.B + bl);
          len = nb > 0 ? __ldg(a.rows + bl) + (nb - 1) * a.n_b : 0;
        }
        int64_t incl = (int64_t)a.H * len;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int64_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += v;
        }
        const int64_t end = base + incl;
        const unsigned hit = __ballot_sync(0xFFFFFFFFu, bl < a.B && end > gpos);
        if (hit) {
          const int l = __ffs(hit) - 1;
          row = bc + l;
          rlen = __shfl_sync(0xFFFFFFFFu, len, l);
          rstart = __shfl_sync(0xFFFFFFFFu, end, l) - (int64_t)a.H * rlen;
        }
        base += __shfl_sync(0xFFFFFFFFu, incl, 31);
      }
      if (row < 0) break;   // past the last token (not reached: gend <= tot)
      const int hh = (int)((gpos - rstart) / rlen);
      const int64_t ustart = rstart + (int64_t)hh * rlen;
      unit = row * a.H + hh;
      c0 = (int)(gpos - ustart);
      c1 = (int)min((int64_t)rlen, gend - ustart);
      sp = gs - (int)(ustart / a.seg_tokens);
      gpos = ustart + c1;
      with_buf = c1 == rlen;
    } else if (n > 0) {
      unit = (int)(gpos / n);
      c0 = (int)(gpos - unit * n);
      c1 = (int)min(n, gend - unit * n);
      sp = gs - (int)((unit * n) / a.seg_tokens);
      gpos = unit * n + c1;
      with_buf = c1 == (int)n && a.n_buf > 0;
    } else {
      unit = gs;
      c0 = c1 = sp = 0;
      gpos = gend;
      with_buf = a.n_buf > 0;
    }
    if (!segment(unit, c0, c1, sp, with_buf)) return;
  }
}

template <typename T, int BITS, int HQ, bool OUT, bool MF, bool KC>
static cudaError_t launch_warp(const DecodeMaps& maps, const DecodeArgs& a, cudaStream_t st) {
  const size_t smem = 1024 + 16 * (size_t)a.tl.cb + 4 * (size_t)a.tl.bytes;
  static std::atomic<int> smem_set[kMaxDevices];   // per device: the limit is a per-device setting
  cudaError_t e = ensure_smem_limit(decode_warp<T, BITS, HQ, OUT, MF, KC>, (int)smem, smem_set);
  if (e != cudaSuccess) return e;
  const int grid = (a.total_splits + 3) / 4;
  decode_warp<T, BITS, HQ, OUT, MF, KC><<<grid, kDThreads, smem, st>>>(maps, a);
  return cudaGetLastError();
}

template <typename T, int BITS, bool MF, bool KC>
static cudaError_t launch_hq(const DecodeMaps& maps, const DecodeArgs& a, cudaStream_t st) {
  switch (a.hq) {
    case 1: return a.k > 0 ? launch_warp<T, BITS, 1, true, MF, KC>(maps, a, st) : launch_warp<T, BITS, 1, false, MF, KC>(maps, a, st);
    case 2: return a.k > 0 ? launch_warp<T, BITS, 2, true, MF, KC>(maps, a, st) : launch_warp<T, BITS, 2, false, MF, KC>(maps, a, st);
    case 4: return a.k > 0 ? launch_warp<T, BITS, 4, true, MF, KC>(maps, a, st) : launch_warp<T, BITS, 4, false, MF, KC>(maps, a, st);
    case 8:
      if constexpr (!KC)   // per-channel key groups: up to 4 query heads per kv head
        return a.k > 0 ? launch_warp<T, BITS, 8, true, MF, KC>(maps, a, st) : launch_warp<T, BITS, 8, false, MF, KC>(maps, a, st);
  }
  return cudaErrorInvalidValue;
}

// binary16 metadata exists for fp16 caches only (the validation rejects it elsewhere)
template <typename T>
static cudaError_t launch_bits(const DecodeMaps& maps, const DecodeArgs& a, cudaStream_t st) {
  constexpr bool kHalf = std::is_same<T, __half>::value;
  if (kHalf && a.meta_f16) {
    switch (a.bits) {
      case 2: return launch_hq<T, 2, kHalf, false>(maps, a, st);
      case 4: return launch_hq<T, 4, kHalf, false>(maps, a, st);
      default: return launch_hq<T, 8, kHalf, false>(maps, a, st);
    }
  }
  switch (a.bits) {
    case 2: return launch_hq<T, 2, false, false>(maps, a, st);
    case 4: return launch_hq<T, 4, false, false>(maps, a, st);
    default: return launch_hq<T, 8, false, false>(maps, a, st);
  }
}

// keys quantized per channel over token groups (16-bit caches, binary32 metadata)
template <typename T>
static cudaError_t launch_bits_kc(const DecodeMaps& maps, const DecodeArgs& a, cudaStream_t st) {
  switch (a.bits) {
    case 2: return launch_hq<T, 2, false, true>(maps, a, st);
    case 4: return launch_hq<T, 4, false, true>(maps, a, st);
    default: return launch_hq<T, 8, false, true>(maps, a, st);
  }
}

}  // namespace gear
