// decode.cu -- decode-step attention over a GEAR-compressed KV cache.
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
// Split-K (flash-decoding style): in decode_warp every warp is one split, a
// run of whole 32-token tiles of one (batch, kv head), for all query heads
// sharing that kv head. It stages tiles of both tensors in its own shared
// memory (asynchronous 16-byte copies, double-buffered), scores with one lane
// per token straight from the packed codes, keeps an online softmax and
// accumulates values with one lane per 4 channels. One extra split per unit
// takes the buffer. decode_combine merges the splits by log-sum-exp.
#include "common.cuh"
#include "decode.cuh"

namespace gear {

constexpr int kDThreads = 128;   // 4 warps, each an independent split
constexpr int kDTile = 32;       // tokens per tile (one per lane)
constexpr int kMaxR = 16;

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

__device__ __forceinline__ int block_of(const DecodeArgs& a, int t) {
  return t < a.blk0_len ? 0 : 1 + (t - a.blk0_len) / a.n_b;
}
__device__ __forceinline__ int block_end(const DecodeArgs& a, int b) {
  return b == 0 ? a.blk0_len : a.blk0_len + b * a.n_b;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Codes as floats without integer conversion. Byte b of a code word is moved
// to mantissa bits 15..22 by one shift; each code of the byte is then masked
// into 1.0f: f = 1 + code * 2^(pos*BITS - 8), pos = index of the code inside
// its byte. The power of two 2^(8 - pos*BITS) is folded into a pre-scaled copy
// of q (keys) or applied once per channel at the end (values), both exact.
template <int BITS>
struct CodeFloats {
  static constexpr int kPerByte = 8 / BITS;
  static constexpr int kPerWord = 32 / BITS;
  // all codes of one 32-bit word, in channel order
  __device__ static __forceinline__ void word(uint32_t w, float (&f)[kPerWord]) {
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int sh = 15 - 8 * b;
      const uint32_t v = sh >= 0 ? (w << sh) : (w >> (-sh));
#pragma unroll
      for (int q = 0; q < kPerByte; ++q) {
        const uint32_t m = ((1u << BITS) - 1u) << (15 + q * BITS);
        f[b * kPerByte + q] = __uint_as_float((v & m) | 0x3F800000u);
      }
    }
  }
  // weight that turns (f - 1) back into the code, for the code at channel c
  __host__ __device__ static constexpr float inv_weight(int c) {
    return (float)(1 << (8 - (c % kPerByte) * BITS));
  }
};

// Stages 32-token tiles of one compressed tensor of one split. The per-token
// arrays of the split's first token are located once; a tile then only adds
// its token offset. Whole, 32-aligned tiles use 16-byte asynchronous copies
// (every region of such a tile is a multiple of 16 bytes and 16-byte
// aligned); other tiles (block tails) use plain loads.
template <typename T, int BITS>
struct Stager {
  static constexpr int W = 4 * BITS;           // code words per token (d = 128)
  static constexpr int kCpr = W / 4;           // 16-byte chunks per code row
  static constexpr int kStride = (W + 4) * 4;  // padded code row in shared memory
  static constexpr int lsz = sizeof(T) == 4 ? 4 : 2;
  const uint8_t* codes;
  const uint8_t* meta;
  const uint8_t* oidx;
  const uint8_t* oval;
  const uint8_t* lf;
  int bm, bi, bo, bl;   // bytes per token of meta, oidx, oval, lf

  __device__ __forceinline__ void init(const CacheView& cv, size_t row0, int G, int k, int rm) {
    bm = G * 8;
    bi = k;
    bo = k * (int)sizeof(T);
    bl = rm * lsz;
    codes = reinterpret_cast<const uint8_t*>(cv.codes) + row0 * W * 4;
    meta = reinterpret_cast<const uint8_t*>(cv.meta) + row0 * bm;
    oidx = cv.oidx + row0 * bi;
    oval = reinterpret_cast<const uint8_t*>(cv.oval) + row0 * bo;
    lf = reinterpret_cast<const uint8_t*>(cv.lfac) + row0 * bl;
  }

  // tokens [dt, dt + nt) of the split into the tile at shared address dst
  __device__ __forceinline__ void stage(const TileLayout& L, uint8_t* dst, int dt, int nt, bool async,
                                        int lane) const {
    if (async) {
      const uint8_t* sc = codes + (size_t)dt * W * 4;
#pragma unroll
      for (int it = 0; it < kCpr; ++it) {
        const int ci = lane + 32 * it;
        const int t = ci / kCpr, jj = ci % kCpr;
        cp_async16(dst + L.codes + t * kStride + jj * 16, sc + ci * 16);
      }
      const uint8_t* sm = meta + (size_t)dt * bm;
      for (int off = lane * 16; off < kDTile * bm; off += 512) cp_async16(dst + L.meta + off, sm + off);
      const uint8_t* si = oidx + (size_t)dt * bi;
      for (int off = lane * 16; off < kDTile * bi; off += 512) cp_async16(dst + L.oidx + off, si + off);
      const uint8_t* so = oval + (size_t)dt * bo;
      for (int off = lane * 16; off < kDTile * bo; off += 512) cp_async16(dst + L.oval + off, so + off);
      const uint8_t* sl = lf + (size_t)dt * bl;
      for (int off = lane * 16; off < kDTile * bl; off += 512) cp_async16(dst + L.lf + off, sl + off);
    } else {
      const uint32_t* sc = reinterpret_cast<const uint32_t*>(codes) + (size_t)dt * W;
      for (int e = lane; e < nt * W; e += 32)
        reinterpret_cast<uint32_t*>(dst + L.codes + (e / W) * kStride)[e % W] = sc[e];
      for (int e = lane; e < nt * bm; e += 32) dst[L.meta + e] = meta[(size_t)dt * bm + e];
      for (int e = lane; e < nt * bi; e += 32) dst[L.oidx + e] = oidx[(size_t)dt * bi + e];
      for (int e = lane; e < nt * bo; e += 32) dst[L.oval + e] = oval[(size_t)dt * bo + e];
      for (int e = lane; e < nt * bl; e += 32) dst[L.lf + e] = lf[(size_t)dt * bl + e];
    }
  }
};

template <typename T>
__device__ __forceinline__ float stage_l(const uint8_t* tile, const TileLayout& L, int t, int j, int rm) {
  if constexpr (sizeof(T) == 4) return reinterpret_cast<const float*>(tile + L.lf)[t * rm + j];
  else return __half2float(reinterpret_cast<const __half*>(tile + L.lf)[t * rm + j]);
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

// Outlier fix-ups of one token: for up to kFast outliers, the channel and the
// difference between the exact value and what codes + low rank give there:
// fix = x_o - (zero_g(c_o) + L_t . Rf[:, c_o]). All loads are issued together.
constexpr int kFast = 4;
template <typename T, int RR>
__device__ __forceinline__ void outlier_fixes(const uint8_t* tile, const TileLayout& L, int t, int k, int G, int rb,
                                              const float (&lt)[RR], const float* rf, int lg, int (&cix)[kFast],
                                              float (&fix)[kFast]) {
  const float2* mt = reinterpret_cast<const float2*>(tile + L.meta) + t * G;
  float xo[kFast], zr[kFast], rv[kFast][RR];
#pragma unroll
  for (int i = 0; i < kFast; ++i) {
    const bool on = i < k;
    cix[i] = on ? tile[L.oidx + t * k + i] : 0;
    xo[i] = on ? (float)reinterpret_cast<const T*>(tile + L.oval)[t * k + i] : 0.0f;
  }
#pragma unroll
  for (int i = 0; i < kFast; ++i) {
    zr[i] = i < k ? mt[cix[i] >> lg].y : 0.0f;
#pragma unroll
    for (int j = 0; j < RR; ++j) rv[i][j] = (i < k && j < rb) ? __ldg(rf + j * 128 + cix[i]) : 0.0f;
  }
#pragma unroll
  for (int i = 0; i < kFast; ++i) {
    float lr = 0.0f;
#pragma unroll
    for (int j = 0; j < RR; ++j) lr = fmaf(lt[j], rv[i][j], lr);
    fix[i] = i < k ? xo[i] - (zr[i] + lr) : 0.0f;
  }
}

// Per-warp shared memory (floats from the warp's base):
//   q [HQ][128] | qw [HQ][128] (q scaled by the code weights) | u [HQ][16]
//   | alr [HQ][16] | w [32][G][HQ] | corr [HQ][128] | accx [HQ][128]
//   | stages: 2 x (K, V tile)
// The [HQ][128] accumulators hold channel c at slot c; loops that touch all
// of them use slot e*32 + lane so that every lane stays in its own bank.
template <typename T, int BITS, int HQ>
__global__ void __launch_bounds__(kDThreads) decode_warp(const DecodeArgs a) {
  extern __shared__ __align__(16) uint8_t dsm[];
  constexpr int W = 4 * BITS;
  constexpr int kStride = Stager<T, BITS>::kStride;
  constexpr int kRReg = 4;   // value low-rank weights kept in registers
  using CF = CodeFloats<BITS>;
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gs = blockIdx.x * 4 + wid;
  if (gs >= a.total_splits) return;
  const int G = a.G, rm = a.r_max, k = a.k;
  const int lg = a.g == 32 ? 5 : (a.g == 64 ? 6 : 7);
  float* q_s = reinterpret_cast<float*>(dsm + (size_t)wid * a.warp_bytes);
  float* qw_s = q_s + HQ * 128;
  float* u_s = qw_s + HQ * 128;
  float* alr_s = u_s + HQ * kMaxR;   // value low-rank weights j >= kRReg
  float* w_s = alr_s + HQ * kMaxR;
  float* corr_s = w_s + kDTile * G * HQ;
  float* accx_s = corr_s + HQ * 128;
  uint8_t* stages = reinterpret_cast<uint8_t*>(accx_s + HQ * 128);
  const TileLayout& L = a.tl;

  const int unit = gs / a.nsplit, sp = gs % a.nsplit;
  const int b = unit / a.H, h = unit % a.H;
  for (int e = lane; e < HQ * 128; e += 32) {
    const float qv = load_elem<T>(a.q, ((size_t)b * a.Hq + (size_t)h * HQ + (e >> 7)) * 128 + (e & 127));
    q_s[e] = qv;
    qw_s[e] = qv * CF::inv_weight(e & 127);
    corr_s[e] = 0.0f;
    accx_s[e] = 0.0f;
  }
  for (int e = lane; e < HQ * kMaxR; e += 32) alr_s[e] = 0.0f;
  __syncwarp();

  // value side: lane owns channels 8*(lane & 15) .. +7 and tokens of parity lane >> 4
  const int lq = lane & 15, par = lane >> 4;
  const int my_g = (8 * lq) >> lg;
  float m[HQ], lsum[HQ], sw[HQ][4], spm[HQ][4], alr[HQ][kRReg];
  uint64_t acc[HQ][4];   // channel pairs (8 channels)
#pragma unroll
  for (int hh = 0; hh < HQ; ++hh) {
    m[hh] = -INFINITY;
    lsum[hh] = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) { acc[hh][e] = 0; sw[hh][e] = 0.0f; spm[hh][e] = 0.0f; alr[hh][e] = 0.0f; }
  }

  if (sp < a.nsplit_comp) {
    // group sums of q and of the weighted q, per 32-channel block
    float qs_blk[HQ][4], qw_blk[HQ][4];
#pragma unroll
    for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
      for (int bk = 0; bk < 4; ++bk) {
        qs_blk[hh][bk] = warp_sum(q_s[hh * 128 + bk * 32 + lane]);
        qw_blk[hh][bk] = warp_sum(qw_s[hh * 128 + bk * 32 + lane]);
      }
    const int c0 = sp * a.chunk;
    const int c1 = min(a.n_comp, c0 + a.chunk);
    // blocks: block 0 = [0, blk0_len), then n_b tokens each; tracked incrementally
    int blk = block_of(a, c0);
    int bend = block_end(a, blk);
    const float* rfk = nullptr;
    const float* rfv = nullptr;
    int rb = 0;
    int t0 = c0, it = 0;
    Stager<T, BITS> sk, sv;
    sk.init(a.K, (size_t)unit * a.n_max + c0, G, k, rm);
    sv.init(a.V, (size_t)unit * a.n_max + c0, G, k, rm);
    // tile [t, min(t + 32, c1, end of its block))
    auto next_end = [&](int t, int be) { return min(min(t + kDTile, c1), be); };
    {
      const int t1 = next_end(t0, bend);
      const bool as = (t1 - t0 == kDTile) && (t0 % kDTile == 0);
      sk.stage(L, stages, t0 - c0, t1 - t0, as, lane);
      sv.stage(L, stages + L.bytes, t0 - c0, t1 - t0, as, lane);
      cp_async_commit();
    }
    int cur_blk = -1;
    while (t0 < c1) {
      if (t0 >= bend) { ++blk; bend = block_end(a, blk); }
      const int t1 = next_end(t0, bend);
      const int nt = t1 - t0;
      uint8_t* tk = stages + (it & 1) * 2 * L.bytes;
      uint8_t* tv = tk + L.bytes;
      if (t1 < c1) {   // prefetch the next tile into the other stage
        const int be2 = t1 >= bend ? block_end(a, blk + 1) : bend;
        const int t2 = next_end(t1, be2);
        const bool as = (t2 - t1 == kDTile) && (t1 % kDTile == 0);
        uint8_t* nk = stages + ((it + 1) & 1) * 2 * L.bytes;
        sk.stage(L, nk, t1 - c0, t2 - t1, as, lane);
        sv.stage(L, nk + L.bytes, t1 - c0, t2 - t1, as, lane);
        cp_async_commit();
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncwarp();

      if (blk != cur_blk) {
        // finish the previous block's value low-rank part, then switch Rf
        if (cur_blk >= 0) {
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
            for (int j = 0; j < kRReg; ++j) alr[hh][j] = warp_sum(alr[hh][j]);
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = e * 32 + lane;
              float v = accx_s[hh * 128 + c];
#pragma unroll
              for (int j = 0; j < kRReg; ++j) if (j < rb) v = fmaf(alr[hh][j], rfv[j * 128 + c], v);
              for (int j = kRReg; j < rb; ++j) v = fmaf(alr_s[hh * kMaxR + j], rfv[j * 128 + c], v);
              accx_s[hh * 128 + c] = v;
            }
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
            for (int j = 0; j < kRReg; ++j) alr[hh][j] = 0.0f;
          __syncwarp();
          for (int e = lane; e < HQ * kMaxR; e += 32) alr_s[e] = 0.0f;
        }
        cur_blk = blk;
        rb = blk == 0 ? a.blk0_rank : a.buffer_rank;
        const size_t rf0 = ((size_t)unit * a.nblk_max + blk) * rm * 128;
        rfk = a.K.rfac + rf0;
        rfv = a.V.rfac + rf0;
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh)
          for (int j = 0; j < rb; ++j) {
            float part = 0.0f;
#pragma unroll
            for (int e = 0; e < 4; ++e) part = fmaf(__ldg(rfk + j * 128 + e * 32 + lane), q_s[hh * 128 + e * 32 + lane], part);
            part = warp_sum(part);
            if (lane == 0) u_s[hh * kMaxR + j] = part;
          }
        __syncwarp();
      }

      // ---------------- scores: lane = token
      const int t = lane;
      const bool live = t < nt;
      float s[HQ];
      {
        const uint32_t* crow = reinterpret_cast<const uint32_t*>(tk + L.codes + t * kStride);
        uint64_t sb[HQ][4][2];   // per 32-channel block, two independent chains
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
          for (int bk = 0; bk < 4; ++bk) { sb[hh][bk][0] = 0; sb[hh][bk][1] = 0; }
#pragma unroll
        for (int j = 0; j < W / 4; ++j) {
          const uint4 wv = *reinterpret_cast<const uint4*>(crow + 4 * j);
          const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
          for (int wi = 0; wi < 4; ++wi) {
            const int cbase = (4 * j + wi) * CF::kPerWord;
            const int bk = cbase >> 5;
            float f[CF::kPerWord];
            CF::word(wd[wi], f);
#pragma unroll
            for (int e = 0; e < CF::kPerWord; e += 4) {
              const int ch = ((cbase + e) >> 2) & 1;
#pragma unroll
              for (int hh = 0; hh < HQ; ++hh) {
                const float4 qv = *reinterpret_cast<const float4*>(qw_s + hh * 128 + cbase + e);
                sb[hh][bk][ch] = fma2(pk2(f[e], f[e + 1]), pk2(qv.x, qv.y), sb[hh][bk][ch]);
                sb[hh][bk][ch] = fma2(pk2(f[e + 2], f[e + 3]), pk2(qv.z, qv.w), sb[hh][bk][ch]);
              }
            }
          }
        }
        const float2* mt = reinterpret_cast<const float2*>(tk + L.meta) + t * G;
        const int bpg = a.g >> 5;   // 32-channel blocks per group
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh) {
          float v = 0.0f;
#pragma unroll
          for (int gi = 0; gi < 4; ++gi) {
            if (gi >= G) break;
            float f = 0.0f, qsw = 0.0f, qss = 0.0f;
#pragma unroll
            for (int bk = 0; bk < 4; ++bk)
              if ((bk / bpg) == gi) {
                f += (lo2(sb[hh][bk][0]) + hi2(sb[hh][bk][0])) + (lo2(sb[hh][bk][1]) + hi2(sb[hh][bk][1]));
                qsw += qw_blk[hh][bk];
                qss += qs_blk[hh][bk];
              }
            const float2 sz = mt[gi];
            v = fmaf(sz.x, f - qsw, v);
            v = fmaf(sz.y, qss, v);
          }
          s[hh] = v;
        }
        if (live) {
          // low-rank part and outlier fix-ups
          float lt[kRReg];
#pragma unroll
          for (int j = 0; j < kRReg; ++j) lt[j] = j < rb ? stage_l<T>(tk, L, t, j, rm) : 0.0f;
#pragma unroll
          for (int j = 0; j < kRReg; ++j)
#pragma unroll
            for (int hh = 0; hh < HQ; ++hh) s[hh] = fmaf(lt[j], j < rb ? u_s[hh * kMaxR + j] : 0.0f, s[hh]);
          for (int j = kRReg; j < rb; ++j) {
            const float lj = stage_l<T>(tk, L, t, j, rm);
#pragma unroll
            for (int hh = 0; hh < HQ; ++hh) s[hh] = fmaf(lj, u_s[hh * kMaxR + j], s[hh]);
          }
          if (k <= kFast && rb <= kRReg) {
            int cix[kFast];
            float fx[kFast];
            outlier_fixes<T, kRReg>(tk, L, t, k, G, rb, lt, rfk, lg, cix, fx);
#pragma unroll
            for (int i = 0; i < kFast; ++i)
#pragma unroll
              for (int hh = 0; hh < HQ; ++hh) s[hh] = fmaf(q_s[hh * 128 + cix[i]], fx[i], s[hh]);
          } else
          for (int i = 0; i < k; ++i) {
            const int c = tk[L.oidx + t * k + i];
            float lr = 0.0f;
#pragma unroll
            for (int j = 0; j < kRReg; ++j) lr = fmaf(lt[j], j < rb ? __ldg(rfk + j * 128 + c) : 0.0f, lr);
            for (int j = kRReg; j < rb; ++j) lr = fmaf(stage_l<T>(tk, L, t, j, rm), __ldg(rfk + j * 128 + c), lr);
            const float xo = (float)reinterpret_cast<const T*>(tk + L.oval)[t * k + i];
            const float fix = xo - (mt[c >> lg].y + lr);
#pragma unroll
            for (int hh = 0; hh < HQ; ++hh) s[hh] = fmaf(q_s[hh * 128 + c], fix, s[hh]);
          }
        }
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh) s[hh] = live ? s[hh] * a.scale_log2 : -INFINITY;
      }

      // ---------------- online softmax (rescale only when the max moved)
      float p[HQ];
#pragma unroll
      for (int hh = 0; hh < HQ; ++hh) {
        const float mnew = fmaxf(m[hh], warp_max(s[hh]));
        p[hh] = live ? exp2f(s[hh] - mnew) : 0.0f;
        if (mnew != m[hh]) {   // warp-uniform
          const float al = exp2f(m[hh] - mnew);
          lsum[hh] *= al;
          const uint64_t al2 = pk2(al, al);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[hh][e] = fma2(acc[hh][e], al2, 0);
            sw[hh][e] *= al;
            spm[hh][e] *= al;
            alr[hh][e] *= al;
            corr_s[hh * 128 + e * 32 + lane] *= al;
            accx_s[hh * 128 + e * 32 + lane] *= al;
          }
          if (rb > kRReg && lane < kMaxR) alr_s[hh * kMaxR + lane] *= al;
        }
        m[hh] = mnew;
        lsum[hh] += p[hh];
      }
      // value-side per-token weights w = p * scale; zero-point and low-rank sums
      {
        const float2* mv = reinterpret_cast<const float2*>(tv + L.meta) + t * G;
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) {
          if (gi >= G) break;
          const float2 sz = live ? mv[gi] : make_float2(0.0f, 0.0f);
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh) {
            const float wv = p[hh] * sz.x;
            w_s[(t * G + gi) * HQ + hh] = wv;
            sw[hh][gi] += wv;
            spm[hh][gi] = fmaf(p[hh], sz.y, spm[hh][gi]);
          }
        }
        if (live) {
#pragma unroll
          for (int j = 0; j < kRReg; ++j) {
            const float lj = j < rb ? stage_l<T>(tv, L, t, j, rm) : 0.0f;
#pragma unroll
            for (int hh = 0; hh < HQ; ++hh) alr[hh][j] = fmaf(p[hh], lj, alr[hh][j]);
          }
          // value outliers
          if (k <= kFast && rb <= kRReg) {
            float lv[kRReg];
#pragma unroll
            for (int j = 0; j < kRReg; ++j) lv[j] = j < rb ? stage_l<T>(tv, L, t, j, rm) : 0.0f;
            int cix[kFast];
            float fx[kFast];
            outlier_fixes<T, kRReg>(tv, L, t, k, G, rb, lv, rfv, lg, cix, fx);
#pragma unroll
            for (int i = 0; i < kFast; ++i)
              if (i < k)
#pragma unroll
                for (int hh = 0; hh < HQ; ++hh) atomicAdd(&corr_s[hh * 128 + cix[i]], p[hh] * fx[i]);
          } else
          for (int i = 0; i < k; ++i) {
            const int c = tv[L.oidx + t * k + i];
            float lr = 0.0f;
#pragma unroll
            for (int j = 0; j < kRReg; ++j)
              lr = fmaf(j < rb ? stage_l<T>(tv, L, t, j, rm) : 0.0f, j < rb ? __ldg(rfv + j * 128 + c) : 0.0f, lr);
            for (int j = kRReg; j < rb; ++j) lr = fmaf(stage_l<T>(tv, L, t, j, rm), __ldg(rfv + j * 128 + c), lr);
            const float xo = (float)reinterpret_cast<const T*>(tv + L.oval)[t * k + i];
            const float fix = xo - (mv[c >> lg].y + lr);
#pragma unroll
            for (int hh = 0; hh < HQ; ++hh) atomicAdd(&corr_s[hh * 128 + c], p[hh] * fix);
          }
        }
      }
      for (int j = kRReg; j < rb; ++j)   // ranks beyond the register slots
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh) {
          const float v = warp_sum(live ? p[hh] * stage_l<T>(tv, L, t, j, rm) : 0.0f);
          if (lane == 0) alr_s[hh * kMaxR + j] += v;
        }
      __syncwarp();

      // ---------------- values: lane = 8 channels, two tokens per step
      {
        const uint8_t* row = tv + L.codes + par * kStride;
        const float* wrow = w_s + (par * G + my_g) * HQ;
#pragma unroll 2
        for (int tt = par; tt < nt; tt += 2) {
          float f[8];
          if constexpr (BITS == 4) {
            CF::word(reinterpret_cast<const uint32_t*>(row)[lq], f);
          } else if constexpr (BITS == 2) {
            float ff[16];
            CF::word(reinterpret_cast<const uint16_t*>(row)[lq], ff);
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = ff[e];
          } else {
            const uint2 ww = reinterpret_cast<const uint2*>(row)[lq];
            float fa[4], fb[4];
            CF::word(ww.x, fa);
            CF::word(ww.y, fb);
#pragma unroll
            for (int e = 0; e < 4; ++e) { f[e] = fa[e]; f[4 + e] = fb[e]; }
          }
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh) {
            const float wv = wrow[hh];
            const uint64_t w2 = pk2(wv, wv);
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[hh][e] = fma2(w2, pk2(f[2 * e], f[2 * e + 1]), acc[hh][e]);
          }
          row += 2 * kStride;
          wrow += 2 * G * HQ;
        }
      }
      __syncwarp();
      t0 = t1;
      ++it;
    }
    // last block's value low-rank part
    if (cur_blk >= 0) {
#pragma unroll
      for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
        for (int j = 0; j < kRReg; ++j) alr[hh][j] = warp_sum(alr[hh][j]);
#pragma unroll
      for (int hh = 0; hh < HQ; ++hh)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = e * 32 + lane;
          float v = accx_s[hh * 128 + c];
#pragma unroll
          for (int j = 0; j < kRReg; ++j) if (j < rb) v = fmaf(alr[hh][j], __ldg(rfv + j * 128 + c), v);
          for (int j = kRReg; j < rb; ++j) v = fmaf(alr_s[hh * kMaxR + j], __ldg(rfv + j * 128 + c), v);
          accx_s[hh * 128 + c] = v;
        }
    }
  } else {
    // ---------------- the streaming buffer: exact tokens, lane = token for keys
    const size_t brow = (size_t)unit * a.n_b;
    for (int t0 = 0; t0 < a.n_buf; t0 += kDTile) {
      const int nt = min(kDTile, a.n_buf - t0);
      const bool live = lane < nt;
      float s[HQ];
#pragma unroll
      for (int hh = 0; hh < HQ; ++hh) s[hh] = 0.0f;
      if (live) {
        for (int c = 0; c < 128; ++c) {
          const float x = load_elem<T>(a.K.buf, (brow + t0 + lane) * 128 + c);
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh) s[hh] = fmaf(x, q_s[hh * 128 + c], s[hh]);
        }
      }
      float p[HQ];
#pragma unroll
      for (int hh = 0; hh < HQ; ++hh) {
        const float sv = live ? s[hh] * a.scale_log2 : -INFINITY;
        const float mnew = fmaxf(m[hh], warp_max(sv));
        const float al = exp2f(m[hh] - mnew);
        m[hh] = mnew;
        p[hh] = live ? exp2f(sv - mnew) : 0.0f;
        lsum[hh] = fmaf(lsum[hh], al, p[hh]);
#pragma unroll
        for (int e = 0; e < 4; ++e) accx_s[hh * 128 + e * 32 + lane] *= al;
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
    float* dst = a.part + (((size_t)b * a.Hq + (size_t)h * HQ + hh) * a.nsplit + sp) * 130;
    if (lane == 0) { dst[0] = m[hh]; dst[1] = l_all; }
    if (par == 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int c = 8 * lq + e;
        dst[2 + c] = CF::inv_weight(c) * (v[e] - swg) + spg + accx_s[hh * 128 + c] + corr_s[hh * 128 + c];
      }
    }
  }
}

template <typename TO>
__global__ void __launch_bounds__(128) decode_combine(const DecodeArgs a) {
  const int bj = blockIdx.x;  // b * Hq + j
  const int c = threadIdx.x;
  const float* p = a.part + (size_t)bj * a.nsplit * 130;
  float M = -INFINITY;
  for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, p[s * 130]);
  float den = 0.0f, num = 0.0f;
  for (int s = 0; s < a.nsplit; ++s) {
    const float m = p[s * 130];
    if (m == -INFINITY) continue;
    const float w = exp2f(m - M);
    den = fmaf(p[s * 130 + 1], w, den);
    num = fmaf(p[s * 130 + 2 + c], w, num);
  }
  const float o = num / den;
  TO* out = reinterpret_cast<TO*>(a.out) + (size_t)bj * 128 + c;
  if constexpr (sizeof(TO) == 4) *out = o;
  else if constexpr (std::is_same<TO, __half>::value) *out = __float2half_rn(o);
  else *out = __float2bfloat16_rn(o);
}

void decode_plan(DecodeArgs& a, int num_sms) {
  const int units = a.B * a.H;
  // per-tensor tile layout in shared memory (16-byte aligned regions)
  auto r16 = [](int x) { return (x + 15) & ~15; };
  const int esz = a.dtype == GEAR_F32 ? 4 : 2;
  TileLayout& L = a.tl;
  L.codes = 0;
  L.meta = L.codes + kDTile * (a.W + 4) * 4;
  L.oidx = L.meta + kDTile * a.G * 8;
  L.oval = L.oidx + r16(kDTile * (a.k > 0 ? a.k : 1));
  L.lf = L.oval + r16(kDTile * (a.k > 0 ? a.k : 1) * esz);
  L.bytes = L.lf + r16(kDTile * a.r_max * (a.dtype == GEAR_F32 ? 4 : 2));
  const int hq = a.hq;
  const int floats = 2 * hq * 128 + 2 * hq * kMaxR + kDTile * a.G * hq + 2 * hq * 128;
  a.warp_bytes = r16(floats * 4) + 4 * L.bytes;
  int nsc = 0;
  if (a.n_comp > 0) {
    // about 48 warps per SM over the whole grid, chunks of whole 32-token tiles
    const long long target = (long long)num_sms * 48;
    long long chunk = ((long long)a.n_comp * units + target - 1) / target;
    chunk = (chunk + kDTile - 1) / kDTile * kDTile;
    if (chunk < 256) chunk = 256;
    a.chunk = (int)chunk;
    nsc = (a.n_comp + a.chunk - 1) / a.chunk;
  } else {
    a.chunk = kDTile;
  }
  a.nsplit_comp = nsc;
  a.nsplit = nsc + (a.n_buf > 0 ? 1 : 0);
  a.total_splits = units * a.nsplit;
}

size_t decode_workspace_bytes(int B, int Hq, int nsplit) { return (size_t)B * Hq * nsplit * 130 * sizeof(float); }

template <typename T, int BITS, int HQ>
static cudaError_t launch_warp(const DecodeArgs& a, cudaStream_t st) {
  const size_t smem = 4 * (size_t)a.warp_bytes;
  static int configured_smem = 0;
  if ((int)smem > configured_smem) {
    cudaError_t e = cudaFuncSetAttribute(decode_warp<T, BITS, HQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    configured_smem = (int)smem;
  }
  const int grid = (a.total_splits + 3) / 4;
  decode_warp<T, BITS, HQ><<<grid, kDThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int BITS>
static cudaError_t launch_hq(const DecodeArgs& a, cudaStream_t st) {
  switch (a.hq) {
    case 1: return launch_warp<T, BITS, 1>(a, st);
    case 2: return launch_warp<T, BITS, 2>(a, st);
    case 4: return launch_warp<T, BITS, 4>(a, st);
    case 8: return launch_warp<T, BITS, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

template <typename T>
static cudaError_t launch_bits(const DecodeArgs& a, cudaStream_t st) {
  switch (a.bits) {
    case 2: return launch_hq<T, 2>(a, st);
    case 4: return launch_hq<T, 4>(a, st);
    default: return launch_hq<T, 8>(a, st);
  }
}

cudaError_t decode_launch(const DecodeArgs& a, cudaStream_t st) {
  cudaError_t e;
  if (a.dtype == GEAR_F16) e = launch_bits<__half>(a, st);
  else if (a.dtype == GEAR_BF16) e = launch_bits<__nv_bfloat16>(a, st);
  else e = launch_bits<float>(a, st);
  if (e != cudaSuccess) return e;
  const int nbj = a.B * a.Hq;
  if (a.out_dtype == GEAR_F32) decode_combine<float><<<nbj, 128, 0, st>>>(a);
  else if (a.out_dtype == GEAR_F16) decode_combine<__half><<<nbj, 128, 0, st>>>(a);
  else decode_combine<__nv_bfloat16><<<nbj, 128, 0, st>>>(a);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ dense
// Test/debug export: reconstruction of every token (compressed, then buffer).
template <typename T, int BITS>
__global__ void __launch_bounds__(128) dense_kernel(const DenseArgs a) {
  const int u = blockIdx.y;
  const int c = threadIdx.x;
  const int ntot = a.n_comp + a.n_buf;
  const int t0 = blockIdx.x * 32;
  constexpr int kPerWord = 32 / BITS;
  for (int t = t0; t < min(t0 + 32, ntot); ++t) {
    float v;
    if (t < a.n_comp) {
      const size_t row = (size_t)u * a.n_max + t;
      const int blk = t < a.blk0_len ? 0 : 1 + (t - a.blk0_len) / a.n_b;
      const int rb = blk == 0 ? a.blk0_rank : a.buffer_rank;
      const uint32_t code = (a.C.codes[row * a.W + c / kPerWord] >> (BITS * (c % kPerWord))) & ((1u << BITS) - 1u);
      const float2 sz = reinterpret_cast<const float2*>(a.C.meta)[row * a.G + c / a.g];
      v = __fmaf_rn((float)code, sz.x, sz.y);
      const float* rf = a.C.rfac + ((size_t)u * a.nblk_max + blk) * a.r_max * 128;
      for (int j = 0; j < rb; ++j) v = fmaf(load_lfac<T>(a.C.lfac, row * a.r_max + j), rf[j * 128 + c], v);
      for (int i = 0; i < a.k; ++i)
        if (a.C.oidx[row * a.k + i] == c) v = load_elem<T>(a.C.oval, row * a.k + i);
    } else {
      v = load_elem<T>(a.C.buf, ((size_t)u * a.n_b + (t - a.n_comp)) * 128 + c);
    }
    a.out[((size_t)u * ntot + t) * 128 + c] = v;
  }
}

template <typename T>
static void launch_dense_t(const DenseArgs& a, dim3 grid, cudaStream_t st) {
  switch (a.bits) {
    case 2: dense_kernel<T, 2><<<grid, 128, 0, st>>>(a); break;
    case 4: dense_kernel<T, 4><<<grid, 128, 0, st>>>(a); break;
    default: dense_kernel<T, 8><<<grid, 128, 0, st>>>(a); break;
  }
}

cudaError_t dense_launch(const DenseArgs& a, cudaStream_t st) {
  const int ntot = a.n_comp + a.n_buf;
  if (ntot == 0) return cudaSuccess;
  dim3 grid((ntot + 31) / 32, a.U);
  if (a.dtype == GEAR_F16) launch_dense_t<__half>(a, grid, st);
  else if (a.dtype == GEAR_BF16) launch_dense_t<__nv_bfloat16>(a, grid, st);
  else launch_dense_t<float>(a, grid, st);
  return cudaGetLastError();
}

}  // namespace gear
