// encode.cu -- GEAR encoder on B200: outliers, group-wise quantization and the
// power-iteration factors of the quantization residual.
//
// Method (GEAR: Efficient KV Cache Compression for LLM Inference, Q3; GEAR: An
// Efficient KV Cache Compression Recipe ..., Cites: SqueezeLLM, FlexGen and
// PowerSGD entries): per token keep the k largest-|x| entries exactly, quantize
// the rest group-wise to b bits (min-max, zero = group minimum), and approximate
// the residual R = X - Dhat of each (batch, head) block with rank-r factors
// from T steps of power iteration started at a seeded matrix Q0.
//
// B200 design. Power iteration only ever touches R through R Q and R^T P, so
// with the d x d Gram matrix M = R^T R (d = 128):
//     P~_t = R Q_{t-1},  P~_t^T P~_t = Q_{t-1}^T M Q_{t-1},  R^T P~_t = M Q_{t-1}.
// Orthonormalizing P~_t by Cholesky-QR of that r x r Gram therefore needs only
// M, and the whole iteration runs on a 128 x 128 matrix. That turns the
// token-long reductions into ONE dense contraction per tile (R_tile^T R_tile,
// tensor cores) and leaves a single extra look at each token at the end
// (L = R Z). Three kernels:
//   E1 encode_quant_gram  persistent, warp-specialized: TMA loads 128-token
//       tiles, 8 quantizer warps compute outliers / codes / metadata (written
//       straight to the cache) and the residual split as bf16 hi + lo, one
//       thread issues tcgen05.mma accumulating hi^T [hi | lo] (M=128, N=256) in
//       tensor memory; per (CTA, unit) segment the partial Gram is written out.
//   E2 encode_power      one CTA per unit: sums the partials in fp64, runs T
//       power steps with Cholesky-QR, writes Rf and Z = Q_{T-1} C_T^-1.
//   E3 encode_lowrank    L = R Z for every token, R rebuilt from the codes.
#include <cuda.h>

#include <cfloat>
#include <cstring>

#include "common.cuh"
#include "encode.cuh"

namespace gear {

// ------------------------------------------------------------------ helpers
// register-pair moves (no integer arithmetic) for the f32x2 operands
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float f2_lo(uint64_t v) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
  return a;
}
__device__ __forceinline__ float f2_hi(uint64_t v) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
  return b;
}
__device__ __forceinline__ uint32_t f2_lo_bits(uint64_t v) {
  uint32_t a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(v));
  return a;
}
__device__ __forceinline__ uint32_t f2_hi_bits(uint64_t v) {
  uint32_t a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(v));
  return b;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// round-to-nearest-even of q in [0, 2^22) by the 1.5 * 2^23 addend: the sum's
// unit in the last place is 1, so the addition itself rounds q to an integer
// (ties to even) and the low mantissa bits of the sum hold it.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr uint32_t kRoundMagicBits = 0x4B400000u;

// Element loads/stores of the KV dtype as 16-bit patterns.
template <typename T>
struct Elem16;
template <>
struct Elem16<__half> {
  static constexpr uint16_t kNaN = 0x7E00;
  __device__ static __half2 hmin(__half2 a, __half2 b) { return __hmin2(a, b); }
  __device__ static __half2 hmax(__half2 a, __half2 b) { return __hmax2(a, b); }
  __device__ static float2 to_f2(uint32_t v) { return __half22float2(*reinterpret_cast<__half2*>(&v)); }
  __device__ static float lo(uint32_t v) { return __half2float(__ushort_as_half((uint16_t)v)); }
  __device__ static uint32_t from_f(float f) { return __half_as_ushort(__float2half_rn(f)); }
};
template <>
struct Elem16<__nv_bfloat16> {
  static constexpr uint16_t kNaN = 0x7FC0;
  __device__ static __nv_bfloat162 hmin(__nv_bfloat162 a, __nv_bfloat162 b) { return __hmin2(a, b); }
  __device__ static __nv_bfloat162 hmax(__nv_bfloat162 a, __nv_bfloat162 b) { return __hmax2(a, b); }
  __device__ static float2 to_f2(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
  }
  __device__ static float lo(uint32_t v) { return __uint_as_float(v << 16); }
  __device__ static uint32_t from_f(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }
};

template <typename T>
__device__ __forceinline__ uint32_t pair_min(uint32_t a, uint32_t b) {
  using V2 = typename std::conditional<std::is_same<T, __half>::value, __half2, __nv_bfloat162>::type;
  V2 r = Elem16<T>::hmin(*reinterpret_cast<V2*>(&a), *reinterpret_cast<V2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
template <typename T>
__device__ __forceinline__ uint32_t pair_max(uint32_t a, uint32_t b) {
  using V2 = typename std::conditional<std::is_same<T, __half>::value, __half2, __nv_bfloat162>::type;
  V2 r = Elem16<T>::hmax(*reinterpret_cast<V2*>(&a), *reinterpret_cast<V2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// Correctly rounded a / s for the code decision. When 2^-100 <= s <= 2^100
// (so s and y = RN(1/s) are normal), the quotient is refined from the
// correctly rounded reciprocal with one exact remainder (Markstein, "Computation
// of elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990: q1 = RN(q0 + r y), r = a - s q0, equals RN(a/s) whenever
// q0 is within one ulp and a/s is normal). Only rint(q) is used and only
// q >= 1/4 can round to a non-zero code, where all operands are normal.
// Otherwise the correctly rounded division intrinsic is used (slow path).
__device__ __forceinline__ uint64_t div_pair_fast(uint64_t a, uint64_t s2n, uint64_t y2) {
  const uint64_t q0 = f2_mul(a, y2);
  const uint64_t r = f2_fma(q0, s2n, a);
  return f2_fma(r, y2, q0);
}
__device__ __forceinline__ uint64_t div_pair_slow(uint64_t a, float s) {
  return f2_pack(__fdiv_rn(f2_lo(a), s), __fdiv_rn(f2_hi(a), s));
}

// ================================================================ E1 ======
// Shared-memory map of E1 (dynamic, 1024-byte aligned):
//   X stages  kNX x kXBytes   TMA tiles, [box][128 rows][128 B] swizzle-128B
//   R stages  kNR x 64 KiB    residual hi (32 KiB) then lo (32 KiB), each two
//                             64-channel blocks of [128 tokens][128 B], swz-128B
//   barriers, tensor-memory slot, abort flag
// For 16-bit inputs two groups of 8 quantizer warps take alternate tiles
// (tile it goes to group it % 2, X stage it % 2 and R stage it % 2), so that
// 16 warps hide each other's latency; fp32 tiles are twice as large and use
// one group. A group hands its X stage back as soon as it has read it, so the
// next tile loads while it quantizes. Every quantizer warp drains every
// segment's accumulator (its share of the columns), so each one waits on
// every phase of the accumulator barriers in order.
constexpr int kTile = 128;       // tokens per tile
constexpr int kQThreads = 256;   // quantizer threads per group (2 per token)
constexpr int kNR = 2;
constexpr uint32_t kRBytes = 65536;

template <typename T>
struct E1Cfg {
  static constexpr int kGroups = sizeof(T) == 4 ? 1 : 2;
  static constexpr int kThreads = 64 + kGroups * kQThreads;
  static constexpr int kNX = kGroups;   // X stage g belongs to group g
  static constexpr uint32_t kXBytes = kTile * 128 * sizeof(T);
  static constexpr int kBoxCols = 128 / sizeof(T);            // 128-byte rows
  static constexpr int kBoxes = 128 / kBoxCols;
  static constexpr uint32_t kBarOff = kNX * kXBytes + kNR * kRBytes;
  static constexpr uint32_t kSmem = kBarOff + 256 + 1024;     // + alignment slack
};

struct XMaps {
  CUtensorMap x[kMaxBatch];   // input rows of each tensor, 128-byte swizzled boxes of 128 rows
};

struct E1Bars {
  uint64_t x_full[2], x_empty[2], r_full[kNR], r_empty[kNR], acc_full, acc_empty, mma_done;
  uint32_t tmem_slot;
  int32_t abort_flag;
};

// byte offset of 16-byte chunk j of row t inside a swizzle-128B box
__device__ __forceinline__ uint32_t swz(int t, int j) { return (uint32_t)(t * 128 + ((j ^ (t & 7)) << 4)); }

__device__ __forceinline__ int64_t seg_first_cta(int64_t tile, int64_t grid, int64_t total) {
  return ((tile + 1) * grid - 1) / total;
}

// One quantizer thread: half h (channels 64h .. 64h+63) of token t of the tile.
// Writes codes/meta/outliers of the token to the cache and the residual split
// into the R stage. `valid` is false for tile rows past the unit's last token.
template <typename T, int BITS, int KMAX>
__device__ __forceinline__ void quantize_half(const EncodeArgs& a, uint8_t* xs, uint8_t* rs, int t, int h,
                                              bool valid, int u, int tok, uint64_t* x_release) {
  constexpr int kCodesPerWord = 32 / BITS;
  constexpr int kWordsHalf = 64 * BITS / 32;
  const float levels = (float)((1 << BITS) - 1);
  const int k = a.k;

  // ---------------- load the half row --------------------------------------
  // 16-bit: 8 chunks of 8 channels (4 packed pairs each); fp32: 16 chunks of 4.
  constexpr int kChunks = sizeof(T) == 4 ? 16 : 8;
  uint32_t xr[32 * (sizeof(T) / 2)];  // 32 pairs (16-bit) or 64 floats (fp32)
  auto chunk_addr = [&](int j) -> uint8_t* {
    if constexpr (sizeof(T) == 4) {
      int box = 2 * h + (j >> 3);
      return xs + box * 16384 + swz(t, j & 7);
    } else {
      return xs + h * 16384 + swz(t, j);
    }
  };
#pragma unroll
  for (int j = 0; j < kChunks; ++j) {
    uint4 v = *reinterpret_cast<const uint4*>(chunk_addr(j));
    xr[4 * j + 0] = v.x; xr[4 * j + 1] = v.y; xr[4 * j + 2] = v.z; xr[4 * j + 3] = v.w;
  }

  // ---------------- outliers: top-k keys (|x|, then lower channel) ---------
  // key = |x| bits << 7 | (127 - c): larger key = larger |x|, ties to the lower
  // channel. Each thread keeps the top KMAX of its 64 keys with a branch-free
  // insertion network, then merges its partner's list (lane ^ 1).
  using Key = typename std::conditional<sizeof(T) == 4, uint64_t, uint32_t>::type;
  Key top[KMAX > 0 ? KMAX : 1];
  int cidx[KMAX > 0 ? KMAX : 1];
  uint32_t oval_bits[KMAX > 0 ? KMAX : 1];
  if constexpr (KMAX > 0) {
#pragma unroll
    for (int i = 0; i < KMAX; ++i) top[i] = 0;
    const uint32_t tb0 = 127u - 64u * h;
#pragma unroll
    for (int e = 0; e < 64; ++e) {
      Key key;
      if constexpr (sizeof(T) == 4) {
        key = ((uint64_t)(xr[e] & 0x7FFFFFFFu) << 7) | (tb0 - e);
      } else {
        uint32_t p = xr[e >> 1];
        uint32_t ab = (e & 1) ? ((p >> 16) & 0x7FFFu) : (p & 0x7FFFu);
        key = (ab << 7) | (tb0 - e);
      }
#pragma unroll
      for (int i = 0; i < KMAX; ++i) {   // one max and one min per level
        const Key hi = max(key, top[i]);
        key = min(key, top[i]);
        top[i] = hi;
      }
    }
    // snapshot the partner's list before either lane modifies its own
    Key other[KMAX];
#pragma unroll
    for (int i = 0; i < KMAX; ++i) other[i] = __shfl_xor_sync(0xFFFFFFFFu, top[i], 1);
#pragma unroll
    for (int i = 0; i < KMAX; ++i) {
      Key key = other[i];
#pragma unroll
      for (int m = 0; m < KMAX; ++m) {
        const Key hi = max(key, top[m]);
        key = min(key, top[m]);
        top[m] = hi;
      }
    }
    // read the k outlier values (both threads read all k), then patch own half
#pragma unroll
    for (int i = 0; i < KMAX; ++i) {
      int c = 127 - (int)(top[i] & 127u);
      cidx[i] = c;
      oval_bits[i] = 0;
      if (i < k && valid) {
        int hh = c >> 6, cl = c & 63;
        uint8_t* p;
        if constexpr (sizeof(T) == 4) {
          p = xs + (2 * hh + (cl >> 5)) * 16384 + swz(t, (cl & 31) >> 2) + (cl & 3) * 4;
          oval_bits[i] = *reinterpret_cast<uint32_t*>(p);
        } else {
          p = xs + hh * 16384 + swz(t, cl >> 3) + (cl & 7) * 2;
          oval_bits[i] = *reinterpret_cast<uint16_t*>(p);
        }
      }
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < KMAX; ++i) {
      int c = cidx[i];
      if (i < k && valid && (c >> 6) == h) {
        int cl = c & 63;
        if constexpr (sizeof(T) == 4) {
          uint8_t* p = xs + (2 * h + (cl >> 5)) * 16384 + swz(t, (cl & 31) >> 2) + (cl & 3) * 4;
          *reinterpret_cast<uint32_t*>(p) = 0x7FC00000u;
        } else {
          uint8_t* p = xs + h * 16384 + swz(t, cl >> 3) + (cl & 7) * 2;
          *reinterpret_cast<uint16_t*>(p) = Elem16<T>::kNaN;
        }
      }
    }
    __syncwarp();
    // reload: outlier slots now hold NaN, which min/max ignore
#pragma unroll
    for (int j = 0; j < kChunks; ++j) {
      uint4 v = *reinterpret_cast<const uint4*>(chunk_addr(j));
      xr[4 * j + 0] = v.x; xr[4 * j + 1] = v.y; xr[4 * j + 2] = v.z; xr[4 * j + 3] = v.w;
    }
  }
  // the X stage is not read again: hand it back to the producer
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(x_release);

  // ---------------- group min / max over non-outliers ----------------------
  // Two 32-channel sub-halves; combined for g >= 64, and with the partner for
  // g = 128. NaN (outlier) operands are ignored by min/max.
  float mn[2], mx[2];
  if constexpr (sizeof(T) == 4) {
#pragma unroll
    for (int sh = 0; sh < 2; ++sh) {
      float lo = __uint_as_float(0x7FC00000u), hi = lo;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        float v = __uint_as_float(xr[32 * sh + e]);
        lo = fminf(lo, v);
        hi = fmaxf(hi, v);
      }
      mn[sh] = lo; mx[sh] = hi;
    }
  } else {
#pragma unroll
    for (int sh = 0; sh < 2; ++sh) {
      uint32_t lo2 = xr[16 * sh], hi2 = xr[16 * sh];
#pragma unroll
      for (int p = 1; p < 16; ++p) {
        lo2 = pair_min<T>(lo2, xr[16 * sh + p]);
        hi2 = pair_max<T>(hi2, xr[16 * sh + p]);
      }
      float2 l = Elem16<T>::to_f2(lo2), u2 = Elem16<T>::to_f2(hi2);
      mn[sh] = fminf(l.x, l.y);
      mx[sh] = fmaxf(u2.x, u2.y);
    }
  }
  if (a.g >= 64) {
    mn[0] = mn[1] = fminf(mn[0], mn[1]);
    mx[0] = mx[1] = fmaxf(mx[0], mx[1]);
  }
  if (a.g == 128) {
    float om = __shfl_xor_sync(0xFFFFFFFFu, mn[0], 1), oM = __shfl_xor_sync(0xFFFFFFFFu, mx[0], 1);
    mn[0] = mn[1] = fminf(mn[0], om);
    mx[0] = mx[1] = fmaxf(mx[0], oM);
  }
  float scale[2], y[2];
  bool fast[2];
#pragma unroll
  for (int sh = 0; sh < 2; ++sh) {
    if (isnan(mn[sh])) { mn[sh] = 0.0f; mx[sh] = 0.0f; }   // group made of outliers only
    mn[sh] = __fadd_rn(mn[sh], 0.0f);                      // -0 -> +0
    mx[sh] = __fadd_rn(mx[sh], 0.0f);
    scale[sh] = __fdiv_rn(__fsub_rn(mx[sh], mn[sh]), levels);
    if (a.meta_f16) {   // stored as binary16; the codes are decided against the stored values
      scale[sh] = __half2float(__float2half_rn(scale[sh]));
      mn[sh] = __fadd_rn(__half2float(__float2half_rn(mn[sh])), 0.0f);
    }
    // scale 0: y = 0 makes the fast path return q = 0 exactly (every code 0)
    fast[sh] = (scale[sh] >= 0x1p-100f && scale[sh] <= 0x1p100f) || scale[sh] == 0.0f;
    y[sh] = scale[sh] == 0.0f ? 0.0f : __frcp_rn(scale[sh]);
  }

  // ---------------- quantize, pack, residual split -------------------------
  uint32_t words[kWordsHalf];
#pragma unroll
  for (int w = 0; w < kWordsHalf; ++w) words[w] = 0u;
  // one pair of channels (2p, 2p + 1); DIV is the division of the pair. The
  // residual split (hi = bf16(R), lo = bf16(R - hi)) comes back packed in ho, lo.
  auto qpair = [&](const int p, const uint64_t mnv, const uint64_t sc2, auto div, uint32_t& ho, uint32_t& lo) {
    const int sh = p >> 4;
    float x0, x1;
    if constexpr (sizeof(T) == 4) {
      x0 = fmaxf(__uint_as_float(xr[2 * p]), mn[sh]);       // NaN -> zero point
      x1 = fmaxf(__uint_as_float(xr[2 * p + 1]), mn[sh]);
    } else {
      uint32_t m2 = Elem16<T>::from_f(mn[sh]);
      m2 |= m2 << 16;
      const float2 f = Elem16<T>::to_f2(pair_max<T>(xr[p], m2));  // NaN -> zero point
      x0 = f.x; x1 = f.y;
    }
    const uint64_t xv = f2_pack(x0, x1);
    const uint64_t av = f2_sub(xv, mnv);
    const uint64_t q = div(av);
    const uint64_t tq = f2_add(q, f2_pack(kRoundMagic, kRoundMagic));
    const uint64_t cf = f2_sub(tq, f2_pack(kRoundMagic, kRoundMagic));
    const uint64_t dh = f2_fma(cf, sc2, mnv);
    const uint64_t rv = f2_sub(xv, dh);
    // pack: word += bits(tq) << (b * e); the constant part of bits(tq) is
    // removed once per word below
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
      const int e = 2 * p + e2;
      const uint32_t bits = e2 ? f2_hi_bits(tq) : f2_lo_bits(tq);
      words[e / kCodesPerWord] += bits << (BITS * (e % kCodesPerWord));
    }
    const __nv_bfloat162 hb = __floats2bfloat162_rn(f2_lo(rv), f2_hi(rv));
    const uint32_t hbits = *reinterpret_cast<const uint32_t*>(&hb);
    const uint64_t hv = f2_pack(__uint_as_float(hbits << 16), __uint_as_float(hbits & 0xFFFF0000u));
    const uint64_t lv = f2_sub(rv, hv);
    const __nv_bfloat162 lb = __floats2bfloat162_rn(f2_lo(lv), f2_hi(lv));
    ho = hbits;
    lo = *reinterpret_cast<const uint32_t*>(&lb);
  };
  // 8 channels (one 16-byte chunk j of the half row) at a time; their residual
  // goes straight to the R stage (MN-major swizzle-128B). Rows past the
  // unit's last token contribute nothing to the Gram.
  auto chunk_out = [&](int j, const uint32_t (&h4)[4], const uint32_t (&l4)[4]) {
    uint8_t* ph = rs + h * 16384 + swz(t, j);
    if (valid) {
      *reinterpret_cast<uint4*>(ph) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
      *reinterpret_cast<uint4*>(ph + 32768) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
    } else {
      *reinterpret_cast<uint4*>(ph) = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(ph + 32768) = make_uint4(0u, 0u, 0u, 0u);
    }
  };
#pragma unroll
  for (int sh = 0; sh < 2; ++sh) {
    const uint64_t mnv = f2_pack(mn[sh], mn[sh]);
    const uint64_t sc2 = f2_pack(scale[sh], scale[sh]);
    if (fast[sh]) {
      const uint64_t y2 = f2_pack(y[sh], y[sh]);
      const uint64_t s2n = f2_pack(-scale[sh], -scale[sh]);
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        uint32_t h4[4], l4[4];
#pragma unroll
        for (int pp = 0; pp < 4; ++pp)
          qpair(16 * sh + 4 * jj + pp, mnv, sc2, [&](uint64_t av) { return div_pair_fast(av, s2n, y2); }, h4[pp],
                l4[pp]);
        chunk_out(4 * sh + jj, h4, l4);
      }
    } else {
      const float sv = scale[sh];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        uint32_t h4[4], l4[4];
#pragma unroll
        for (int pp = 0; pp < 4; ++pp)
          qpair(16 * sh + 4 * jj + pp, mnv, sc2, [&](uint64_t av) { return div_pair_slow(av, sv); }, h4[pp], l4[pp]);
        chunk_out(4 * sh + jj, h4, l4);
      }
    }
  }
  {
    uint32_t magic_sum = 0;
#pragma unroll
    for (int e = 0; e < kCodesPerWord; ++e) magic_sum += kRoundMagicBits << (BITS * e);
#pragma unroll
    for (int w = 0; w < kWordsHalf; ++w) words[w] -= magic_sum;
  }

  // ---------------- cache outputs -------------------------------------------
  if (valid) {
    const EncodeTensor& ten = a.ten[u / a.Uper];
    const size_t row = (size_t)(u % a.Uper) * a.n_max + (size_t)(a.t_off + tok);
    uint32_t* cw = ten.codes + row * a.W + h * kWordsHalf;
#pragma unroll
    for (int w = 0; w < kWordsHalf; w += 4)
      *reinterpret_cast<uint4*>(cw + w) = make_uint4(words[w], words[w + 1], words[w + 2], words[w + 3]);
    // meta: (scale, zero) per group; this thread owns groups in its half
    const int gsz = a.g;
    auto put_meta = [&](int gi, float sc, float z) {
      if (a.meta_f16) reinterpret_cast<__half2*>(ten.meta)[row * a.G + gi] = __floats2half2_rn(sc, z);   // exact
      else reinterpret_cast<float2*>(ten.meta)[row * a.G + gi] = make_float2(sc, z);
    };
    if (gsz == 32) {
      put_meta(2 * h, scale[0], mn[0]);
      put_meta(2 * h + 1, scale[1], mn[1]);
    } else if (gsz == 64) {
      put_meta(h, scale[0], mn[0]);
    } else if (h == 0) {
      put_meta(0, scale[0], mn[0]);
    }
    if constexpr (KMAX > 0) {
      if (h == 0 && k > 0) {
        // ascending channel order: selection by rank among the k channels
        uint8_t* oi = ten.oidx + row * k;
#pragma unroll
        for (int i = 0; i < KMAX; ++i) {
          if (i < k) {
            int rank = 0;
#pragma unroll
            for (int m = 0; m < KMAX; ++m) rank += (m < k && cidx[m] < cidx[i]) ? 1 : 0;
            oi[rank] = (uint8_t)cidx[i];
            if constexpr (sizeof(T) == 4)
              reinterpret_cast<uint32_t*>(ten.oval)[row * k + rank] = oval_bits[i];
            else
              reinterpret_cast<uint16_t*>(ten.oval)[row * k + rank] = (uint16_t)oval_bits[i];
          }
        }
      }
    }
  }
}

template <typename T, int BITS, int KMAX>
__global__ void __launch_bounds__(E1Cfg<T>::kThreads, 1)
    encode_quant_gram(const __grid_constant__ XMaps maps, const EncodeArgs a) {
  using C = E1Cfg<T>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint8_t* xst = smem;
  uint8_t* rst = smem + C::kNX * C::kXBytes;
  E1Bars* bars = reinterpret_cast<E1Bars*>(smem + C::kBarOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t total = a.total_tiles;
  const int64_t grid = gridDim.x;
  const int64_t t_begin = (int64_t)blockIdx.x * total / grid;
  const int64_t t_end = ((int64_t)blockIdx.x + 1) * total / grid;
  const int ntiles = (int)(t_end - t_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kNX; ++s) { mbar_init(&bars->x_full[s], 1); mbar_init(&bars->x_empty[s], 8); }
    for (int s = 0; s < kNR; ++s) { mbar_init(&bars->r_full[s], 8); mbar_init(&bars->r_empty[s], 1); }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, C::kGroups * 8);
    mbar_init(&bars->mma_done, 1);
    bars->abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem_slot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;

  auto is_seg_start = [&](int64_t i) { return i == t_begin || (i % a.tpu) == 0; };
  auto is_seg_end = [&](int64_t i) { return i + 1 == t_end || ((i + 1) % a.tpu) == 0; };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int last_it[2] = {-1, -1};
      for (int it = 0; it < ntiles; ++it) {
        const int s = it % C::kNX;
        if (!mbar_wait(&bars->x_empty[s], ((it / C::kNX) & 1) ^ 1)) { bars->abort_flag = 1; break; }
        const int64_t tile = t_begin + it;
        const int u = (int)(tile / a.tpu);
        const int t0 = (int)(tile % a.tpu) * kTile;
        const int32_t row0 = (u % a.Uper) * a.n + t0;
        const CUtensorMap* xm = &maps.x[u / a.Uper];
        mbar_arrive_expect_tx(&bars->x_full[s], C::kXBytes);
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_2d(xst + s * C::kXBytes + b * 16384, xm, &bars->x_full[s], b * C::kBoxCols, row0);
        last_it[s] = it;
      }
      // every issued load must have landed before the CTA may exit
      for (int s = 0; s < C::kNX; ++s)
        if (last_it[s] >= 0) mbar_wait(&bars->x_full[s], (last_it[s] / C::kNX) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_f16(128, 256, true, true, true);
      int seg = 0;
      for (int it = 0; it < ntiles; ++it) {
        const int64_t tile = t_begin + it;
        const int sr = it % kNR;
        bool ok = mbar_wait(&bars->r_full[sr], (it / kNR) & 1);
        const bool first = is_seg_start(tile);
        if (ok && first) ok = mbar_wait(&bars->acc_empty, (seg & 1) ^ 1);
        if (!ok) { bars->abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t base = smem_u32(rst + sr * kRBytes);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          uint64_t ad = smem_desc_sw128(base + kk * 2048, 16384, 1024);
          uint64_t bd = smem_desc_sw128(base + kk * 2048, 16384, 1024);
          tc_mma_f16(tmem, ad, bd, kIdesc, (first && kk == 0) ? 0u : 1u);
        }
        tc_commit(&bars->r_empty[sr]);
        if (is_seg_end(tile)) { tc_commit(&bars->acc_full); ++seg; }
      }
      // every MMA this thread issued has completed before tensor memory is freed
      tc_commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0);
    }
  } else {
    // ------------------------------------------------ quantizer warps
    const int group = (warp - 2) >> 3;
    const int qid = (threadIdx.x - 64) & (kQThreads - 1);
    const int t = qid >> 1, h = qid & 1;
    // drain share: TMEM lanes of quarter warp & 3, output columns [col0, col0 + ncol)
    constexpr int kNcol = 128 / (2 * C::kGroups);
    const int quarter = warp & 3;
    const int col0 = ((warp - 2) >> 2) * kNcol;
    // segments of this CTA: S = 0 .. nseg-1, one per unit its tiles touch
    const int64_t u_first = t_begin / a.tpu;
    const int nseg = ntiles > 0 ? (int)((t_end - 1) / a.tpu - u_first + 1) : 0;
    int drained = 0;   // segments drained by this warp
    // drains, in order, every segment that ended at tile index <= upto
    auto drain = [&](int upto) -> bool {
      while (drained < nseg) {
        const int64_t end_tile = min(t_end, (u_first + drained + 1) * (int64_t)a.tpu) - 1;
        if (end_tile > t_begin + upto) return true;
        if (!mbar_wait(&bars->acc_full, drained & 1)) return false;
        tc_fence_after();
        const int ue = (int)(end_tile / a.tpu);
        const int ch = quarter * 32 + lane;
        const int64_t slot = (int64_t)blockIdx.x - seg_first_cta((int64_t)ue * a.tpu, grid, total);
        float* dst = a.gram + (((int64_t)ue * a.maxc + slot) * 128 + ch) * 128;
        const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
#pragma unroll
        for (int cc = 0; cc < kNcol; cc += 32) {
          uint32_t d1[32], d2[32];
          tmem_ld_32x32b_x32(lane_addr + col0 + cc, d1);
          tmem_ld_32x32b_x32(lane_addr + 128 + col0 + cc, d2);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            float4 v;
            v.x = __uint_as_float(d1[j + 0]) + 2.0f * __uint_as_float(d2[j + 0]);
            v.y = __uint_as_float(d1[j + 1]) + 2.0f * __uint_as_float(d2[j + 1]);
            v.z = __uint_as_float(d1[j + 2]) + 2.0f * __uint_as_float(d2[j + 2]);
            v.w = __uint_as_float(d1[j + 3]) + 2.0f * __uint_as_float(d2[j + 3]);
            *reinterpret_cast<float4*>(dst + col0 + cc + j) = v;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->acc_empty);
        ++drained;
      }
      return true;
    };
    bool ok = true;
    for (int it = 0; it < ntiles && ok; ++it) {
      const int64_t tile = t_begin + it;
      if (it % C::kGroups != group) continue;
      const int u = (int)(tile / a.tpu);
      const int t0 = (int)(tile % a.tpu) * kTile;
      const int s = it % C::kNX, sr = it % kNR;
      ok = mbar_wait(&bars->x_full[s], (it / C::kNX) & 1);
      ok = ok && mbar_wait(&bars->r_empty[sr], ((it / kNR) & 1) ^ 1);
      if (!ok || bars->abort_flag) { ok = false; break; }
      quantize_half<T, BITS, KMAX>(a, xst + s * C::kXBytes, rst + sr * kRBytes, t, h, t0 + t < a.n, u, t0 + t,
                                   &bars->x_empty[s]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->r_full[sr]);
      ok = drain(it);
    }
    if (ok) ok = drain(ntiles - 1);
    if (!ok) bars->abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ================================================================ E2 ======
// Per unit: M = sym(sum of partial Grams), then T power steps with
// Cholesky-QR on the r x r Gram. Outputs Rf (cache, scaled 2^-e) and
// Z = Q_{T-1} C_T^-1 scaled 2^e (workspace) so that E3's R Z is the stored L.
// The partials arrive by 64 KiB bulk asynchronous copies, two in flight, and
// are summed in a fixed order (deterministic); M is kept in fp32 (the
// partials carry about 17 significant bits), products accumulate in fp64.
constexpr int kE2Threads = 512;
constexpr int kE2Parts = kE2Threads / 128;   // threads per row of W = M Q
constexpr int kMStride = 132;  // padded fp32 row of M

__device__ __forceinline__ uint64_t splitmix64_at(uint64_t seed, uint64_t i) {
  // output number i (0-based) of the splitmix64 stream whose state starts at seed
  uint64_t z = seed + (i + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <int RM>
struct E2Smem {
  float M[128 * kMStride];
  double Q[128 * RM];
  uint64_t bar[2];
  union {
    float stage[2][16384];   // partial Grams in flight (phase 1)
    struct {                 // power-iteration scratch (phase 2)
      double Wp[kE2Parts * 128 * RM];
      double red[4 * RM * RM];
      double Xi[RM * RM];
    } it;
  } u;
};

template <int RM>
__global__ void __launch_bounds__(kE2Threads, 1) encode_power(const EncodeArgs a) {
  extern __shared__ __align__(128) uint8_t sm2raw[];
  E2Smem<RM>& S = *reinterpret_cast<E2Smem<RM>*>(sm2raw);
  const int u = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = a.r;
  const int64_t total = a.total_tiles, grid = a.grid_e1;
  const int64_t c0 = seg_first_cta((int64_t)u * a.tpu, grid, total);
  const int64_t c1 = seg_first_cta((int64_t)u * a.tpu + a.tpu - 1, grid, total);
  const int nseg = (int)(c1 - c0 + 1);
  const float* part = a.gram + (int64_t)u * a.maxc * 16384;

  if (tid == 0) {
    mbar_init(&S.bar[0], 1);
    mbar_init(&S.bar[1], 1);
    fence_mbarrier_init();
    for (int sg = 0; sg < 2 && sg < nseg; ++sg) {
      mbar_arrive_expect_tx(&S.bar[sg], 65536);
      bulk_load(S.u.stage[sg], part + (int64_t)sg * 16384, 65536, &S.bar[sg]);
    }
  }
  // Q0 from the seed (columns r .. RM-1 stay zero)
  for (int e = tid; e < 128 * RM; e += kE2Threads) {
    const int i = e / RM, j = e % RM;
    double v = 0.0;
    if (j < r) {
      const uint64_t z = splitmix64_at(a.seed, (uint64_t)(i * r + j));
      v = (double)(uint32_t)(z >> 40) * 0x1p-23 - 1.0;
    }
    S.Q[e] = v;
  }
  __syncthreads();
  for (int sg = 0; sg < nseg; ++sg) {
    const int b = sg & 1;
    // a wait that gives up (error word set) ends the unit: no factors are
    // computed from an incomplete Gram; the other stage's copy, if one was
    // issued, is given its own bounded wait so that nothing lands after exit
    if (!__syncthreads_and(mbar_wait(&S.bar[b], (sg >> 1) & 1))) {
      if (tid == 0 && sg + 1 < nseg) mbar_wait(&S.bar[b ^ 1], ((sg + 1) >> 1) & 1);
      __syncthreads();
      return;
    }
    for (int e4 = tid; e4 < 4096; e4 += kE2Threads) {
      const float4 v = reinterpret_cast<const float4*>(S.u.stage[b])[e4];
      float4* dst = reinterpret_cast<float4*>(&S.M[(e4 >> 5) * kMStride + ((e4 & 31) << 2)]);   // 16-byte aligned rows
      if (sg == 0) {
        *dst = v;
      } else {
        const float4 o = *dst;
        *dst = make_float4(o.x + v.x, o.y + v.y, o.z + v.z, o.w + v.w);
      }
    }
    __syncthreads();
    if (tid == 0 && sg + 2 < nseg) {
      mbar_arrive_expect_tx(&S.bar[b], 65536);
      bulk_load(S.u.stage[b], part + (int64_t)(sg + 2) * 16384, 65536, &S.bar[b]);
    }
  }
  for (int e = tid; e < 128 * 128; e += kE2Threads) {
    const int i = e >> 7, j = e & 127;
    if (i < j) {
      const float mv = 0.5f * (S.M[i * kMStride + j] + S.M[j * kMStride + i]);
      S.M[i * kMStride + j] = mv;
      S.M[j * kMStride + i] = mv;
    }
  }
  __syncthreads();

  const int i = tid & 127, wpart = tid >> 7;
  for (int step = 0; step < a.T; ++step) {
    // W = M Q: kE2Parts threads per row, each over 128 / kE2Parts channels
    {
      double w[RM];
#pragma unroll
      for (int j = 0; j < RM; ++j) w[j] = 0.0;
#pragma unroll 8
      for (int c = wpart * (128 / kE2Parts); c < (wpart + 1) * (128 / kE2Parts); ++c) {
        const double mv = (double)S.M[c * kMStride + i];
#pragma unroll
        for (int j = 0; j < RM; ++j) w[j] = fma(mv, S.Q[c * RM + j], w[j]);
      }
#pragma unroll
      for (int j = 0; j < RM; ++j) S.u.it.Wp[(wpart * 128 + i) * RM + j] = w[j];
    }
    __syncthreads();
    // G = Q^T W (upper triangle), reduced by warp then across warps
    if (tid < 128) {
      double w[RM], qv[RM];
#pragma unroll
      for (int j = 0; j < RM; ++j) {
        double v = S.u.it.Wp[i * RM + j];
#pragma unroll
        for (int pp = 1; pp < kE2Parts; ++pp) v += S.u.it.Wp[(pp * 128 + i) * RM + j];
        w[j] = v;
        qv[j] = S.Q[i * RM + j];
      }
#pragma unroll
      for (int j = 0; j < RM; ++j) S.u.it.Wp[i * RM + j] = w[j];
#pragma unroll
      for (int p = 0; p < RM; ++p)
#pragma unroll
        for (int q = p; q < RM; ++q) {
          double v = qv[p] * w[q];
          for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
          if (lane == 0) S.u.it.red[(warp * RM + p) * RM + q] = v;
        }
    }
    __syncthreads();
    if (tid == 0) {
      // Cholesky G = C^T C (upper C) with column dropping, then X = C^-1 so
      // that P~ X has orthonormal (or zero) columns. All indices are
      // compile-time, so C and X stay in registers.
      double C[RM][RM], X[RM][RM], rinv[RM];
      bool nz[RM];
#pragma unroll
      for (int p = 0; p < RM; ++p)
#pragma unroll
        for (int q = 0; q < RM; ++q) {
          double g = 0.0;
          if (p <= q) g = S.u.it.red[p * RM + q] + S.u.it.red[(RM + p) * RM + q] + S.u.it.red[(2 * RM + p) * RM + q] +
                          S.u.it.red[(3 * RM + p) * RM + q];
          C[p][q] = g;
          X[p][q] = 0.0;
        }
#pragma unroll
      for (int j = 0; j < RM; ++j) {
        const double gjj = C[j][j];
#pragma unroll
        for (int m2 = 0; m2 < j; ++m2) {
          double v = C[m2][j];
#pragma unroll
          for (int i2 = 0; i2 < m2; ++i2) v -= C[i2][m2] * C[i2][j];
          C[m2][j] = v * rinv[m2];   // 0 for a dropped column
        }
        double piv = gjj;
#pragma unroll
        for (int m2 = 0; m2 < j; ++m2) piv -= C[m2][j] * C[m2][j];
        nz[j] = j < r && gjj > 0.0 && piv > 1e-10 * gjj;
        // one reciprocal square root per column gives both C_jj and 1 / C_jj
        const double rs = nz[j] ? rsqrt(piv) : 0.0;
        C[j][j] = nz[j] ? piv * rs : 1.0;
        rinv[j] = rs;
      }
#pragma unroll
      for (int j = 0; j < RM; ++j) {
        const double inv = rinv[j];
#pragma unroll
        for (int i2 = 0; i2 <= j; ++i2) {
          double v = (i2 == j) ? 1.0 : 0.0;
#pragma unroll
          for (int m2 = 0; m2 < j; ++m2) v -= C[m2][j] * X[i2][m2];
          X[i2][j] = v * inv;
        }
      }
#pragma unroll
      for (int p = 0; p < RM; ++p)
#pragma unroll
        for (int q = 0; q < RM; ++q) S.u.it.Xi[p * RM + q] = X[p][q];
    }
    __syncthreads();
    const bool last = (step + 1 == a.T);
    if (tid < 128) {
      double zq[RM], wq[RM];
#pragma unroll
      for (int j = 0; j < RM; ++j) {
        double sq = 0.0, swv = 0.0;
#pragma unroll
        for (int m2 = 0; m2 < RM; ++m2) {
          sq = fma(S.Q[i * RM + m2], S.u.it.Xi[m2 * RM + j], sq);
          swv = fma(S.u.it.Wp[i * RM + m2], S.u.it.Xi[m2 * RM + j], swv);
        }
        zq[j] = sq;
        wq[j] = swv;
      }
      if (!last) {
        // row i is read and written by this thread only
#pragma unroll
        for (int j = 0; j < RM; ++j) S.Q[i * RM + j] = wq[j];
      } else {
        const double sL = ldexp(1.0, a.e_blk), sR = ldexp(1.0, -a.e_blk);
        // Z rows in channel pairs: zbuf[u][i / 2][j][i % 2], the layout E3 copies in one piece
        float* zrow = a.zbuf + (((int64_t)u * 64 + (i >> 1)) * 16) * 2 + (i & 1);
#pragma unroll
        for (int j = 0; j < 16; ++j) zrow[2 * j] = (j < RM && j < r) ? (float)(zq[j < RM ? j : 0] * sL) : 0.0f;
        const int rp = rpad_of(a.r_max);
        float* rrow = a.ten[u / a.Uper].rfac + (((int64_t)(u % a.Uper) * a.nblk_max + a.blk) * 128 + i) * rp;
        for (int j = 0; j < rp; ++j) {
          double wv = 0.0;
#pragma unroll
          for (int jj = 0; jj < RM; ++jj) if (jj == j) wv = wq[jj];
          rrow[j] = j < r ? (float)(wv * sR) : 0.0f;
        }
      }
    }
    __syncthreads();
  }
}

// ================================================================ E3 ======
// L rows: L_t = R_t Z for every token of the block, with R rebuilt as
// x - fma(code, scale, zero) on every slot; the outlier slots' contribution
// (x_o - zero) Z[c_o] is then removed again (their residual is 0).
// One CTA per 128-token tile of one unit, one thread per token. The tile's
// input rows (the encoder's tensor map: 128-byte swizzled boxes), code rows
// (16-byte-chunk swizzle) and, for G >= 2, meta rows arrive by tensor copies
// on one mbarrier; several CTAs per SM overlap one tile's copies with another
// tile's arithmetic. A thread accumulates channel pairs in f32x2 registers.
// Codes become floats by the mantissa trick f = 1 + code * 2^-w (w = 8 - pos
// * bits for the code at position pos of its byte), so that
// fma(f - 1, scale * 2^w, zero) is exactly fma(code, scale, zero) as long as
// scale * 2^8 is finite; a token with a larger scale takes a plain loop.
constexpr int kE3Threads = 128;

struct E3Maps {
  // per tensor: input rows, cache code rows, cache meta rows (G >= 2)
  CUtensorMap x[kMaxBatch], codes[kMaxBatch], meta[kMaxBatch];
};

template <typename T, int BITS, int RMAX>
struct E3Cfg {
  static constexpr int kXB = kTile * 128 * (int)sizeof(T);   // input tile
  static constexpr int kRow = 16 * BITS;                     // code bytes per token
  static constexpr int kCB = kTile * kRow;                   // code tile
  static constexpr int kMB = kTile * 32;                     // meta tile (G <= 4)
  static constexpr int kZOff = kXB + kCB + kMB;              // Z pairs [64][16] float2
  static constexpr int kZBytes = 64 * 16 * 8;
  static constexpr int kBarOff = kZOff + kZBytes;
  static constexpr int kSmem = kBarOff + 16 + 1024;          // + alignment slack
};

template <int R>
__device__ __forceinline__ int swz_rows(int t) {   // chunk swizzle of R-byte rows (R = 32, 64, 128)
  return ((t * R) >> 7) & (R / 16 - 1);
}

template <typename T, int BITS, int RMAX>
__global__ void __launch_bounds__(kE3Threads, 4) encode_lowrank(const __grid_constant__ E3Maps maps, const EncodeArgs a) {
  using C = E1Cfg<T>;
  using F = E3Cfg<T, BITS, RMAX>;
  constexpr int W = 4 * BITS;
  constexpr int kPerByte = 8 / BITS;
  extern __shared__ uint8_t e3raw[];
  uint8_t* sm = align_smem_1024(e3raw);
  uint8_t* xs = sm;
  uint8_t* cs = sm + F::kXB;
  uint8_t* ms = cs + F::kCB;
  float2* Zp = reinterpret_cast<float2*>(sm + F::kZOff);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + F::kBarOff);
  const int u = blockIdx.y, t0 = blockIdx.x * kTile, t = threadIdx.x;
  const int G = a.G, k = a.k, r = a.r;
  const int mrb = meta_row_bytes(G, a.meta_f16);   // meta bytes per token
  const bool meta_tma = mrb >= 16;
  const int lg = a.g == 32 ? 5 : (a.g == 64 ? 6 : 7);
  const int tn = u / a.Uper, ul = u % a.Uper;
  const EncodeTensor& ten = a.ten[tn];
  const int crow = ul * a.n_max + a.t_off + t0;   // cache row of the tile's first token
  if (t == 0) {
    mbar_init(bar, 1);
    fence_mbarrier_init();
    mbar_arrive_expect_tx(bar, (uint32_t)(F::kXB + F::kCB + F::kZBytes + (meta_tma ? kTile * mrb : 0)));
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(Zp)),
                 "l"(a.zbuf + (int64_t)u * (F::kZBytes / 4)), "r"((uint32_t)F::kZBytes), "r"(smem_u32(bar))
                 : "memory");
    for (int b = 0; b < C::kBoxes; ++b) tma_load_2d(xs + b * 16384, &maps.x[tn], bar, b * C::kBoxCols, ul * a.n + t0);
    tma_load_2d(cs, &maps.codes[tn], bar, 0, crow);
    if (meta_tma) tma_load_2d(ms, &maps.meta[tn], bar, 0, crow);
  }
  // Zp[p][j] = (Z[2p][j], Z[2p + 1][j]) arrives with the tile (E2 writes it in this layout)
  const bool valid = t0 + t < a.n;
  const size_t row = (size_t)crow + t;
  // short meta rows (under 16 bytes) come straight from global memory
  float2 szr[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
  if (!meta_tma && valid) {
    if (a.meta_f16) {
      const __half2* mh = reinterpret_cast<const __half2*>(ten.meta) + row * G;
      szr[0] = __half22float2(mh[0]);
      if (G == 2) szr[1] = __half22float2(mh[1]);
    } else {
      szr[0] = reinterpret_cast<const float2*>(ten.meta)[row];
    }
  }
  // the token's first outliers, fetched while the tile is in flight
  constexpr int kOF = 4;
  int oc[kOF];
  float ox[kOF];
#pragma unroll
  for (int i = 0; i < kOF; ++i) {
    const bool on = valid && i < k;
    oc[i] = on ? ten.oidx[row * k + i] : 0;
    if constexpr (sizeof(T) == 4) ox[i] = on ? reinterpret_cast<const float*>(ten.oval)[row * k + i] : 0.0f;
    else ox[i] = on ? Elem16<T>::lo(reinterpret_cast<const uint16_t*>(ten.oval)[row * k + i]) : 0.0f;
  }
  __syncthreads();
  const bool landed = mbar_wait(bar, 0);
  if (!landed || !valid) return;

  // this token's meta row: fp32 group gi at byte (8 gi) ^ mx (32-byte rows
  // swizzled), binary16 group gi at byte 4 gi
  const uint8_t* mrow = ms + t * mrb;
  const int mx = mrb == 32 ? ((t >> 2) & 1) << 4 : 0;
  auto group = [&](int gi) -> float2 {
    if (!meta_tma) return gi == 0 ? szr[0] : szr[1];
    if (a.meta_f16) return __half22float2(*reinterpret_cast<const __half2*>(mrow + 4 * gi));
    return *reinterpret_cast<const float2*>(mrow + ((gi << 3) ^ mx));
  };
  bool big = false;
  for (int gi = 0; gi < G; ++gi) big |= !(group(gi).x <= 0x1p100f);
  // the code words of 32 channels [32 q, 32 q + 32): 4*BITS bytes of the row
  auto codes32 = [&](int q, uint32_t (&cw)[BITS]) {
    const uint8_t* rowp = cs + t * F::kRow;
    if constexpr (BITS == 2) {
      const uint2 v = *reinterpret_cast<const uint2*>(rowp + ((((q >> 1) ^ swz_rows<F::kRow>(t)) << 4) | ((q & 1) << 3)));
      cw[0] = v.x; cw[1] = v.y;
    } else {
#pragma unroll
      for (int h = 0; h < BITS / 4; ++h) {
        const uint4 v = *reinterpret_cast<const uint4*>(rowp + (((BITS / 4 * q + h) ^ swz_rows<F::kRow>(t)) << 4));
        cw[4 * h] = v.x; cw[4 * h + 1] = v.y; cw[4 * h + 2] = v.z; cw[4 * h + 3] = v.w;
      }
    }
  };

  uint64_t acc[RMAX];
#pragma unroll
  for (int j = 0; j < RMAX; ++j) acc[j] = 0;
  // 8 channels [8 jb, 8 jb + 8) of the input row, as floats
  auto xblock = [&](int jb, float (&xv)[8]) {
    if constexpr (sizeof(T) == 4) {
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        const uint4 v = *reinterpret_cast<const uint4*>(xs + (jb >> 2) * 16384 + swz(t, 2 * (jb & 3) + hq));
        xv[4 * hq] = __uint_as_float(v.x); xv[4 * hq + 1] = __uint_as_float(v.y);
        xv[4 * hq + 2] = __uint_as_float(v.z); xv[4 * hq + 3] = __uint_as_float(v.w);
      }
    } else {
      const uint4 v = *reinterpret_cast<const uint4*>(xs + (jb >> 3) * 16384 + swz(t, jb & 7));
      const uint32_t pr[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = Elem16<T>::to_f2(pr[q]);
        xv[2 * q] = f.x; xv[2 * q + 1] = f.y;
      }
    }
  };
  if (!big) {
    const uint32_t one = a.one_bits;
    const uint64_t one2 = f2_pack(1.0f, 1.0f);
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {   // 32 channels per pass, one group (g >= 32)
      uint32_t cw[BITS];
      codes32(q, cw);
      const float2 sz = group((32 * q) >> lg);
      const uint64_t sc2 = f2_pack(sz.x, sz.x), zr2 = f2_pack(sz.y, sz.y);
#pragma unroll
      for (int bq = 0; bq < 4; ++bq) {
        const int jb = 4 * q + bq;
        float xv[8];
        xblock(jb, xv);
        float f[8];   // the block's 8 codes as 1 + code * 2^-w
        if constexpr (BITS == 4) {
          CodeFloats<4>::word(cw[bq], f, one);
        } else if constexpr (BITS == 2) {
          float ff[16];
          CodeFloats<2>::word(cw[bq >> 1] >> (16 * (bq & 1)), ff, one);
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = ff[e];
        } else {
          float fa[4], fb[4];
          CodeFloats<8>::word(cw[2 * bq], fa, one);
          CodeFloats<8>::word(cw[2 * bq + 1], fb, one);
#pragma unroll
          for (int e = 0; e < 4; ++e) { f[e] = fa[e]; f[4 + e] = fb[e]; }
        }
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const int cl = 2 * p;   // channel inside the block; 8*jb is a whole number of bytes
          const uint64_t w2 = f2_pack((float)(1 << (8 - (cl % kPerByte) * BITS)),
                                      (float)(1 << (8 - ((cl + 1) % kPerByte) * BITS)));
          const uint64_t cf = f2_sub(f2_pack(f[cl], f[cl + 1]), one2);
          const uint64_t dh = f2_fma(cf, f2_mul(sc2, w2), zr2);
          const uint64_t rr = f2_sub(f2_pack(xv[cl], xv[cl + 1]), dh);
          const float4* zq = reinterpret_cast<const float4*>(Zp + (4 * jb + p) * 16);
#pragma unroll
          for (int j = 0; j < RMAX; j += 2) {
            const float4 z = zq[j >> 1];
            acc[j] = f2_fma(rr, f2_pack(z.x, z.y), acc[j]);
            acc[j + 1] = f2_fma(rr, f2_pack(z.z, z.w), acc[j + 1]);
          }
        }
      }
    }
  } else {
    constexpr int kCpw = 32 / BITS;
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
      uint32_t cw[BITS];
      codes32(q, cw);
      const float2 sz = group((32 * q) >> lg);
#pragma unroll
      for (int bq = 0; bq < 4; ++bq) {
        const int jb = 4 * q + bq;
        float xv[8];
        xblock(jb, xv);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          float rr[2];
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int c = 8 * bq + 2 * p + e2;   // channel inside the 32
            const float code = (float)((cw[c / kCpw] >> (BITS * (c % kCpw))) & ((1u << BITS) - 1u));
            rr[e2] = __fsub_rn(xv[2 * p + e2], __fmaf_rn(code, sz.x, sz.y));
          }
          const uint64_t rv = f2_pack(rr[0], rr[1]);
#pragma unroll
          for (int j = 0; j < RMAX; ++j)
            acc[j] = f2_fma(rv, *reinterpret_cast<const uint64_t*>(&Zp[(4 * jb + p) * 16 + j]), acc[j]);
        }
      }
    }
  }
  // outlier slots: their residual is zero; remove what the loop added
  for (int i = 0; i < k; ++i) {
    int c;
    float x;
    if (i < kOF) {
#pragma unroll
      for (int i2 = 0; i2 < kOF; ++i2)
        if (i2 == i) { c = oc[i2]; x = ox[i2]; }
    } else {
      c = ten.oidx[row * k + i];
      if constexpr (sizeof(T) == 4) x = reinterpret_cast<const float*>(ten.oval)[row * k + i];
      else x = Elem16<T>::lo(reinterpret_cast<const uint16_t*>(ten.oval)[row * k + i]);
    }
    const float2 sz = group(c >> lg);
    const float rr = __fsub_rn(x, __fmaf_rn(0.0f, sz.x, sz.y));
#pragma unroll
    for (int j = 0; j < RMAX; ++j) {
      const float2 z = Zp[(c >> 1) * 16 + j];
      const float v = rr * ((c & 1) ? z.y : z.x);
      acc[j] = f2_sub(acc[j], (c & 1) ? f2_pack(0.0f, v) : f2_pack(v, 0.0f));
    }
  }
  for (int q = 0; q < a.r_max; ++q) {
    float v = 0.0f;
#pragma unroll
    for (int j = 0; j < RMAX; ++j)
      if (j == q) v = f2_lo(acc[j]) + f2_hi(acc[j]);
    if (q >= r) v = 0.0f;
    if constexpr (sizeof(T) == 4) reinterpret_cast<float*>(ten.lfac)[row * a.r_max + q] = v;
    else reinterpret_cast<__half*>(ten.lfac)[row * a.r_max + q] = __float2half_rn(v);
  }
}

// ================================================================ host =====
template <typename T, int BITS, int KMAX>
static cudaError_t launch_e1(const XMaps& map, const EncodeArgs& a, int grid, cudaStream_t st) {
  auto kern = encode_quant_gram<T, BITS, KMAX>;
  static std::atomic<int> smem_set[kMaxDevices];   // per device: the limit is a per-device setting
  cudaError_t e = ensure_smem_limit(kern, E1Cfg<T>::kSmem, smem_set);
  if (e != cudaSuccess) return e;
  kern<<<grid, E1Cfg<T>::kThreads, E1Cfg<T>::kSmem, st>>>(map, a);
  return cudaGetLastError();
}

template <typename T, int BITS>
static cudaError_t launch_e1_k(const XMaps& map, const EncodeArgs& a, int grid, cudaStream_t st) {
  if (a.k == 0) return launch_e1<T, BITS, 0>(map, a, grid, st);
  if (a.k == 3) return launch_e1<T, BITS, 3>(map, a, grid, st);
  if (a.k <= 4) return launch_e1<T, BITS, 4>(map, a, grid, st);
  if (a.k <= 8) return launch_e1<T, BITS, 8>(map, a, grid, st);
  return launch_e1<T, BITS, 16>(map, a, grid, st);
}

template <typename T>
static cudaError_t launch_e1_b(const XMaps& map, const EncodeArgs& a, int grid, cudaStream_t st) {
  switch (a.bits) {
    case 2: return launch_e1_k<T, 2>(map, a, grid, st);
    case 4: return launch_e1_k<T, 4>(map, a, grid, st);
    default: return launch_e1_k<T, 8>(map, a, grid, st);
  }
}

template <typename T, int BITS, int RMAX>
static cudaError_t launch_e3(const E3Maps& maps, const EncodeArgs& a, dim3 grid, cudaStream_t st) {
  auto kern = encode_lowrank<T, BITS, RMAX>;
  constexpr int smem = E3Cfg<T, BITS, RMAX>::kSmem;
  static std::atomic<int> smem_set[kMaxDevices];
  cudaError_t e = ensure_smem_limit(kern, smem, smem_set);
  if (e != cudaSuccess) return e;
  kern<<<grid, kE3Threads, smem, st>>>(maps, a);
  return cudaGetLastError();
}

template <typename T, int BITS>
static cudaError_t launch_e3_r(const E3Maps& maps, const EncodeArgs& a, dim3 grid, cudaStream_t st) {
  if (a.r <= 4) return launch_e3<T, BITS, 4>(maps, a, grid, st);
  if (a.r <= 8) return launch_e3<T, BITS, 8>(maps, a, grid, st);
  return launch_e3<T, BITS, 16>(maps, a, grid, st);
}

template <typename T>
static cudaError_t launch_e3_b(const E3Maps& maps, const EncodeArgs& a, cudaStream_t st) {
  dim3 grid(a.tpu, a.U);
  switch (a.bits) {
    case 2: return launch_e3_r<T, 2>(maps, a, grid, st);
    case 4: return launch_e3_r<T, 4>(maps, a, grid, st);
    default: return launch_e3_r<T, 8>(maps, a, grid, st);
  }
}

PFN_encodeTiled tensor_map_encoder() {
  static PFN_encodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  }
  return fn;
}

int encode_grid(const EncodeArgs& a, int num_sms) {
  int64_t total = a.total_tiles;
  return (int)(total < num_sms ? total : num_sms);
}

int encode_maxc(int64_t total_tiles, int grid, int tpu) {
  int64_t tmin = total_tiles / grid;
  if (tmin < 1) tmin = 1;
  int64_t m = (tpu - 1 + tmin - 1) / tmin + 1;
  if (m > tpu) m = tpu;
  if (m > grid) m = grid;
  return (int)m;
}

cudaError_t encode_launch(EncodeArgs a, int num_sms, cudaStream_t st) {
  const int esz = a.dtype == GEAR_F32 ? 4 : 2;
  PFN_encodeTiled enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  // x: [Uper * n rows][128], boxes of 128 bytes x 128 rows, 128-byte swizzle
  E3Maps m3;
  memset(&m3, 0, sizeof(m3));
  const CUtensorMapDataType dt = a.dtype == GEAR_F32   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : a.dtype == GEAR_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                        : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const uint64_t crows = (uint64_t)a.Uper * a.n_max;
  for (int tn = 0; tn < a.nt; ++tn) {
    const cuuint64_t dims[2] = {128, (cuuint64_t)a.Uper * (cuuint64_t)a.n};
    const cuuint64_t strides[1] = {(cuuint64_t)128 * esz};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)kTile};
    const cuuint32_t estr[2] = {1, 1};
    CUresult cr = enc(&m3.x[tn], dt, 2, const_cast<void*>(a.ten[tn].kv), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
    if (!cache_row_map(enc, &m3.codes[tn], a.ten[tn].codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.W, crows, kTile))
      return cudaErrorInvalidValue;
    const int mrb = meta_row_bytes(a.G, a.meta_f16);
    if (mrb >= 16 &&
        !cache_row_map(enc, &m3.meta[tn], a.ten[tn].meta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, mrb / 4, crows, kTile))
      return cudaErrorInvalidValue;
  }
  XMaps xm;
  memcpy(xm.x, m3.x, sizeof(xm.x));

  const int grid = a.grid_e1;
  cudaError_t e;
  if (a.dtype == GEAR_F16) e = launch_e1_b<__half>(xm, a, grid, st);
  else if (a.dtype == GEAR_BF16) e = launch_e1_b<__nv_bfloat16>(xm, a, grid, st);
  else e = launch_e1_b<float>(xm, a, grid, st);
  if (e != cudaSuccess) return e;
  if (a.r == 0) return cudaSuccess;

  {
    const int RM = a.r <= 4 ? 4 : (a.r <= 8 ? 8 : 16);
    const size_t sm2 = RM == 4 ? sizeof(E2Smem<4>) : (RM == 8 ? sizeof(E2Smem<8>) : sizeof(E2Smem<16>));
    auto kern = RM == 4 ? encode_power<4> : (RM == 8 ? encode_power<8> : encode_power<16>);
    static std::atomic<int> smem_set[3][kMaxDevices];
    e = ensure_smem_limit(kern, (int)sm2, smem_set[RM == 4 ? 0 : (RM == 8 ? 1 : 2)]);
    if (e != cudaSuccess) return e;
    kern<<<a.U, kE2Threads, sm2, st>>>(a);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  if (a.dtype == GEAR_F16) return launch_e3_b<__half>(m3, a, st);
  if (a.dtype == GEAR_BF16) return launch_e3_b<__nv_bfloat16>(m3, a, st);
  return launch_e3_b<float>(m3, a, st);
}

}  // namespace gear
