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
__device__ __forceinline__ uint64_t div_pair_slow2(uint64_t a, float s0, float s1) {
  return f2_pack(__fdiv_rn(f2_lo(a), s0), __fdiv_rn(f2_hi(a), s1));
}

// Barrier among `count` threads (whole warps) under id (1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
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
  // per-channel key groups: per quantizer group, the column min/max partials
  // [4 x 32-token blocks][64 channel pairs] (2 KB), then the channels'
  // (zero, scale, 1/scale, fast) of up to 4 token groups (8 KB)
  static constexpr uint32_t kChOff = kBarOff + 256;
  static constexpr uint32_t kChBytes = 10240;
  static constexpr uint32_t kSmemCh = kSmem + kGroups * kChBytes;
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

// ---------------------------------------------------------------- top-k
// Packed 16-bit helpers on |x| bit patterns (non-negative finite fp16/bf16
// magnitudes order like their bit patterns read as unsigned integers).
__device__ __forceinline__ uint32_t umax2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// 0xFFFF in each half whose magnitude is >= the threshold's (same half)
template <typename T>
__device__ __forceinline__ uint32_t ge_mask2(uint32_t a, uint32_t th2) {
  uint32_t r;
  if constexpr (std::is_same<T, __half>::value) asm("set.ge.u32.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(th2));
  else asm("set.ge.u32.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(th2));
  return r;
}
// Sorts 8 values into descending order (19 compare-exchanges, the optimal
// network for 8 inputs; Knuth, TAOCP vol. 3, 5.3.4).
template <typename K>
__device__ __forceinline__ void sort8_desc(K (&v)[8]) {
  constexpr int kNet[19][2] = {{0, 1}, {2, 3}, {4, 5}, {6, 7}, {0, 2}, {1, 3}, {4, 6}, {5, 7}, {1, 2}, {5, 6},
                               {0, 4}, {3, 7}, {1, 5}, {2, 6}, {1, 4}, {3, 6}, {2, 4}, {3, 5}, {3, 4}};
#pragma unroll
  for (int i = 0; i < 19; ++i) {
    const K a = v[kNet[i][0]], b = v[kNet[i][1]];
    v[kNet[i][0]] = max(a, b);
    v[kNet[i][1]] = min(a, b);
  }
}

// Merges two descending lists of 8 into the 8 largest of both, descending:
// the elementwise maxima against the reversed second list are the 8 largest as
// a bitonic sequence (Batcher's half-cleaner), which a bitonic merger sorts.
template <typename K>
__device__ __forceinline__ void merge8_desc(K (&a)[8], const K (&b)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = max(a[i], b[7 - i]);
  constexpr int kMerge[12][2] = {{0, 4}, {1, 5}, {2, 6}, {3, 7}, {0, 2}, {1, 3},
                                 {4, 6}, {5, 7}, {0, 1}, {2, 3}, {4, 5}, {6, 7}};
#pragma unroll
  for (int i = 0; i < 12; ++i) {
    const K x = a[kMerge[i][0]], y = a[kMerge[i][1]];
    a[kMerge[i][0]] = max(x, y);
    a[kMerge[i][1]] = min(x, y);
  }
}

// Candidates of the per-token top-k for 16-bit inputs (k <= 8): a lower bound
// theta on the token's k-th largest |x| that costs a few operations per pair,
// then the exact selection over the few entries with |x| >= theta only.
// Bound: split the token into 16 blocks of 8 channels (8 per half); the k
// largest block maxima are k distinct entries, so the k-th largest block
// maximum is <= the token's k-th largest |x|. Every entry of the top k (|x| >=
// k-th largest) is therefore a candidate. Returns the candidates of this half as
// two bit words: bit p of w[i] <-> channel 2(16i + p), bit 16 + p <-> channel
// 2(16i + p) + 1.
template <typename T>
__device__ __forceinline__ void topk_candidates(const uint32_t (&xr)[32], int k, bool valid, uint32_t (&w)[2]) {
  uint32_t ab[32];
#pragma unroll
  for (int p = 0; p < 32; ++p) ab[p] = xr[p] & 0x7FFF7FFFu;
  uint32_t bm[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t m = umax2(umax2(ab[4 * j], ab[4 * j + 1]), umax2(ab[4 * j + 2], ab[4 * j + 3]));
    bm[j] = max(m & 0xFFFFu, m >> 16);
  }
  sort8_desc(bm);
  uint32_t other[8];   // the partner half's sorted block maxima
#pragma unroll
  for (int i = 0; i < 8; ++i) other[i] = __shfl_xor_sync(0xFFFFFFFFu, bm[i], 1);
  merge8_desc(bm, other);
  uint32_t th = bm[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) th = (i == k - 1) ? bm[i] : th;
  const uint32_t th2 = th | (th << 16);
  w[0] = w[1] = 0u;
#pragma unroll
  for (int p = 0; p < 32; ++p) w[p >> 4] |= ge_mask2<T>(ab[p], th2) & (0x00010001u << (p & 15));
  if (!valid) w[0] = w[1] = 0u;   // rows past the unit's end select nothing
}

// One quantizer thread: half h (channels 64h .. 64h+63) of token t of the tile.
// Writes codes/meta/outliers of the token to the cache and the residual split
// into the R stage. `valid` is false for tile rows past the unit's last token.
template <typename T, int BITS, int KMAX, bool CH>
__device__ __forceinline__ void quantize_half(const EncodeArgs& a, uint8_t* xs, uint8_t* rs, int t, int h,
                                              bool valid, int u, int tok, uint64_t* x_release, uint8_t* chs,
                                              int group, int t0) {
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
    auto insert = [&](Key key) {
#pragma unroll
      for (int i = 0; i < KMAX; ++i) {   // one max and one min per level
        const Key hi = max(key, top[i]);
        key = min(key, top[i]);
        top[i] = hi;
      }
    };
    if constexpr (sizeof(T) == 2 && KMAX <= 8) {
      // filtered: only the candidates of topk_candidates enter the insertion
      uint32_t cw[2];
      topk_candidates<T>(xr, k, valid, cw);
      const uint8_t* xh = xs + h * 16384;
      while ((cw[0] | cw[1]) != 0u) {
        const bool lo = cw[0] != 0u;
        const uint32_t wv = lo ? cw[0] : cw[1];
        const int b = __ffs(wv) - 1;
        if (lo) cw[0] = wv & (wv - 1u); else cw[1] = wv & (wv - 1u);
        const int e = ((((lo ? 0 : 16) + (b & 15)) << 1) | (b >> 4));   // channel inside the half
        const uint32_t ab = *reinterpret_cast<const uint16_t*>(xh + swz(t, e >> 3) + (e & 7) * 2) & 0x7FFFu;
        insert((Key)((ab << 7) | (tb0 - e)));
      }
    } else {
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
        insert(key);
      }
    }
    // snapshot the partner's list before either lane modifies its own
    Key other[KMAX];
#pragma unroll
    for (int i = 0; i < KMAX; ++i) other[i] = __shfl_xor_sync(0xFFFFFFFFu, top[i], 1);
    if constexpr (KMAX == 8) {
      merge8_desc(top, other);   // both lists are sorted descending
    } else {
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
  if constexpr (!CH) {
    // the X stage is not read again: hand it back to the producer
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(x_release);
  }

  // ---------------- per-channel key groups (KIVI-combined) -----------------
  // Every channel gets its own (zero, scale) over each group of g consecutive
  // tokens; the tile's 128 rows (outlier slots now NaN, which min/max ignore)
  // are read column-wise by the group's 256 threads, one channel pair and one
  // 32-token block each, after all rows are patched.
  float4* prm = reinterpret_cast<float4*>(chs + 2048);
  if constexpr (CH) {
    const int qid = 2 * t + h;
    uint2* part = reinterpret_cast<uint2*>(chs);
    named_barrier_sync(1 + group, kQThreads);
    {
      const int cp = qid & 63, sb = qid >> 6;
      const int nval = min(a.n - t0, kTile);
      const uint32_t nan2 = (uint32_t)Elem16<T>::kNaN * 0x10001u;
      uint32_t lo2 = nan2, hi2 = nan2;
      const uint8_t* col = xs + (cp >> 5) * 16384 + (cp & 3) * 4;
      for (int r = 32 * sb; r < 32 * sb + 32; ++r) {
        if (r >= nval) break;
        const uint32_t v = *reinterpret_cast<const uint32_t*>(col + swz(r, (cp & 31) >> 2));
        lo2 = pair_min<T>(lo2, v);
        hi2 = pair_max<T>(hi2, v);
      }
      part[sb * 64 + cp] = make_uint2(lo2, hi2);
    }
    named_barrier_sync(1 + group, kQThreads);
    // the X stage is not read again: hand it back to the producer
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(x_release);
    {
      const int ng = kTile / a.g, sbg = a.g / 32;
      const EncodeTensor& ten = a.ten[u / a.Uper];
      const size_t slot_row = ((size_t)(u % a.Uper) * a.ch_slots + a.slot0 + t0 / a.g) * 128;
      for (int e = qid; e < ng * 128; e += kQThreads) {
        const int j = e >> 7, c = e & 127;
        float mnc = __uint_as_float(0x7FC00000u), mxc = mnc;
        for (int sb = j * sbg; sb < (j + 1) * sbg; ++sb) {
          const uint2 pr = part[sb * 64 + (c >> 1)];
          const float2 l = Elem16<T>::to_f2(pr.x), hv = Elem16<T>::to_f2(pr.y);
          mnc = fminf(mnc, (c & 1) ? l.y : l.x);
          mxc = fmaxf(mxc, (c & 1) ? hv.y : hv.x);
        }
        if (isnan(mnc)) { mnc = 0.0f; mxc = 0.0f; }   // no non-outlier entry
        mnc = __fadd_rn(mnc, 0.0f);                    // -0 -> +0
        mxc = __fadd_rn(mxc, 0.0f);
        const float sc = __fdiv_rn(__fsub_rn(mxc, mnc), levels);
        const bool fst = (sc >= 0x1p-100f && sc <= 0x1p100f) || sc == 0.0f;
        prm[j * 128 + c] = make_float4(mnc, sc, sc == 0.0f ? 0.0f : __frcp_rn(sc), fst ? 1.0f : 0.0f);
        if (t0 + j * a.g < a.n)   // a group with tokens of this block: its meta to the cache
          reinterpret_cast<float2*>(ten.meta)[slot_row + (size_t)j * 128 + c] = make_float2(sc, mnc);
      }
    }
    named_barrier_sync(1 + group, kQThreads);
  }

  // ---------------- group min / max over non-outliers ----------------------
  // Two 32-channel sub-halves; combined for g >= 64, and with the partner for
  // g = 128. NaN (outlier) operands are ignored by min/max.
  float mn[2] = {0.0f, 0.0f}, mx[2] = {0.0f, 0.0f};
  if constexpr (CH) {
  } else if constexpr (sizeof(T) == 4) {
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
  if (!CH && a.g >= 64) {
    mn[0] = mn[1] = fminf(mn[0], mn[1]);
    mx[0] = mx[1] = fmaxf(mx[0], mx[1]);
  }
  if (!CH && a.g == 128) {
    float om = __shfl_xor_sync(0xFFFFFFFFu, mn[0], 1), oM = __shfl_xor_sync(0xFFFFFFFFu, mx[0], 1);
    mn[0] = mn[1] = fminf(mn[0], om);
    mx[0] = mx[1] = fmaxf(mx[0], oM);
  }
  float scale[2] = {0.0f, 0.0f}, y[2] = {0.0f, 0.0f};
  bool fast[2] = {true, true};
#pragma unroll
  for (int sh = 0; sh < 2 && !CH; ++sh) {
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
    float x0, x1;
    if constexpr (sizeof(T) == 4) {
      x0 = fmaxf(__uint_as_float(xr[2 * p]), f2_lo(mnv));       // NaN -> zero point
      x1 = fmaxf(__uint_as_float(xr[2 * p + 1]), f2_hi(mnv));
    } else {
      const uint32_t m2 = Elem16<T>::from_f(f2_lo(mnv)) | (Elem16<T>::from_f(f2_hi(mnv)) << 16);
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
  if constexpr (CH) {
    // per channel: the (zero, scale, 1/scale) of the token's group
    const float4* pj = prm + (t / a.g) * 128 + 64 * h;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      uint32_t h4[4], l4[4];
#pragma unroll
      for (int pp = 0; pp < 4; ++pp) {
        const int p = 4 * jj + pp;
        const float4 P0 = pj[2 * p], P1 = pj[2 * p + 1];
        const uint64_t mnv = f2_pack(P0.x, P1.x), sc2 = f2_pack(P0.y, P1.y);
        if (P0.w != 0.0f && P1.w != 0.0f) {
          const uint64_t y2 = f2_pack(P0.z, P1.z), s2n = f2_pack(-P0.y, -P1.y);
          qpair(p, mnv, sc2, [&](uint64_t av) { return div_pair_fast(av, s2n, y2); }, h4[pp], l4[pp]);
        } else {
          qpair(p, mnv, sc2, [&](uint64_t av) { return div_pair_slow2(av, P0.y, P1.y); }, h4[pp], l4[pp]);
        }
      }
      chunk_out(jj, h4, l4);
    }
  }
#pragma unroll
  for (int sh = 0; sh < 2 && !CH; ++sh) {
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
    if (CH) {
      // per-channel groups: the meta was written by the column pass
    } else if (gsz == 32) {
      put_meta(2 * h, scale[0], mn[0]);
      put_meta(2 * h + 1, scale[1], mn[1]);
    } else if (gsz == 64) {
      put_meta(h, scale[0], mn[0]);
    } else if (h == 0) {
      put_meta(0, scale[0], mn[0]);
    }
    if constexpr (KMAX > 0 && KMAX <= 8) {
      // ascending channel order: sort (channel, value bits) keys by channel
      // (unused slots sort last); half 0 stores the channels, half 1 the values
      using SK = typename std::conditional<sizeof(T) == 4, uint64_t, uint32_t>::type;
      constexpr int kSh = sizeof(T) == 4 ? 32 : 16;
      SK sk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        sk[i] = (i < KMAX && i < k) ? (((SK)cidx[i < KMAX ? i : 0] << kSh) | (SK)oval_bits[i < KMAX ? i : 0]) : ~(SK)0;
      if constexpr (KMAX <= 4) {
        constexpr int kNet4[5][2] = {{0, 1}, {2, 3}, {0, 2}, {1, 3}, {1, 2}};   // optimal network for 4
#pragma unroll
        for (int i = 0; i < 5; ++i) {
          const SK x = sk[kNet4[i][0]], y = sk[kNet4[i][1]];
          sk[kNet4[i][0]] = min(x, y);
          sk[kNet4[i][1]] = max(x, y);
        }
      } else {
        sort8_desc(sk);   // descending; read back from the end
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const SK x = sk[i];
          sk[i] = sk[7 - i];
          sk[7 - i] = x;
        }
      }
      if (h == 0) {
        uint8_t* oi = ten.oidx + row * k;
#pragma unroll
        for (int i = 0; i < KMAX; ++i)
          if (i < k) oi[i] = (uint8_t)(sk[i] >> kSh);
      } else {
#pragma unroll
        for (int i = 0; i < KMAX; ++i) {
          if (i < k) {
            if constexpr (sizeof(T) == 4) reinterpret_cast<uint32_t*>(ten.oval)[row * k + i] = (uint32_t)sk[i];
            else reinterpret_cast<uint16_t*>(ten.oval)[row * k + i] = (uint16_t)sk[i];
          }
        }
      }
    } else if constexpr (KMAX > 0) {
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

template <typename T, int BITS, int KMAX, bool CH>
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
      quantize_half<T, BITS, KMAX, CH>(a, xst + s * C::kXBytes, rst + sr * kRBytes, t, h, t0 + t < a.n, u, t0 + t,
                                       &bars->x_empty[s], smem + C::kChOff + group * C::kChBytes, group, t0);
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

// Channel held by element e of 16-byte chunk m of the spread-code image.
template <int BITS>
__device__ __forceinline__ int spread_channel(int m, int e) {
  if constexpr (BITS == 4) return 8 * m + (e >> 1) + 4 * (e & 1);            // word m: codes i, i + 4
  else if constexpr (BITS == 2) return 16 * (m >> 1) + 4 * (m & 1) + (e >> 1) + 8 * (e & 1);   // i, i + 8
  else return 8 * m + 4 * (e >> 2) + 2 * (e & 1) + ((e >> 1) & 1);         // bytes 0, 2 then 1, 3
}

// Position (chunk, element) of channel c in the spread-code image (inverse of
// spread_channel).
__host__ __device__ inline void spread_position(int bits, int c, int& m, int& el) {
  const int i = c & 7;
  if (bits == 4) {
    m = c >> 3;
    el = 2 * (i & 3) + (i >> 2);
  } else if (bits == 2) {
    const int w = c & 15;
    m = 2 * (c >> 4) + ((w & 7) >> 2);
    el = 2 * (w & 3) + (w >> 3);
  } else {
    const int r = i & 3;
    m = c >> 3;
    el = 4 * (i >> 2) + 2 * (r & 1) + (r >> 1);
  }
}

// Z (d x r, r <= 16) as a B operand of E3's tensor-core products, K-major
// (channels contiguous): element (row n, channel c) of one 16-bit part of N
// rows sits in box c / 64 (N * 128 bytes), row n, 16-byte chunk
// ((c % 64) / 8) ^ (n % 8) (the 128-byte swizzle), byte 2 (c % 8).
__host__ __device__ constexpr int zimg_offset(int N, int n, int c) {
  return (c >> 6) * (N * 128) + n * 128 + ((((c & 63) >> 3) ^ (n & 7)) << 4) + ((c & 7) << 1);
}

// ================================================================ E2 ======
// Per unit: M = sym(sum of partial Grams), then T power steps with
// Cholesky-QR on the r x r Gram. Outputs Rf (cache, scaled 2^-e) and
// Z = Q_{T-1} C_T^-1 scaled 2^e (workspace) so that E3's R Z is the stored L.
// The partials are read by 16-byte loads, all of a partial's in flight at
// once, and summed in a fixed order (deterministic); M is kept in fp32 (the
// partials carry about 17 significant bits), products accumulate in fp64.
// NT threads per CTA: 512 when the units fit in one wave (more threads per
// unit), else 256 with two CTAs per SM (about 95 KB of shared memory at
// r <= 8), so that one unit's serial steps (the r x r factorization on one
// thread) overlap another unit's products.
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

template <int RM, int NT>
struct E2Smem {
  float M[128 * kMStride];
  double Q[128 * RM];
  struct {   // power-iteration scratch
    double Wp[NT / 128 * 128 * RM];
    double red[4 * RM * RM];
    double Xi[RM * RM];
  } it;
};

// The unit's slab for E3 (see kZSlab): fp32 Z rows, then for 16-bit inputs
// the operand images of X Z (16 rows, fp16 hi + lo or bf16 hi + mid + lo) and
// of C Z (block-diagonal, the codes' spread order, fp16 hi + lo), both scaled
// by 2^-sh so that max |Z| 2^-sh lies in [8, 16), with S_g (sums of the fp16
// parts over each group) and the scales; for fp32 inputs the bf16 hi + lo
// image of R Z (unscaled). Zf [128][16] holds Z on entry; Vf [128][16] is
// scratch. Called by all threads of the block.
__device__ void write_z_slab(const EncodeArgs& a, int u, const float* Zf, float* Vf) {
  const int tid = threadIdx.x, nth = blockDim.x;
  uint8_t* slab = reinterpret_cast<uint8_t*>(a.zbuf) + (int64_t)u * kZSlab;
  float* rows = reinterpret_cast<float*>(slab + kSlabRows);
  for (int e = tid; e < 128 * 16; e += nth) rows[e] = Zf[e];
  __shared__ float red[32];
  float m = 0.0f;
  for (int e = tid; e < 128 * 16; e += nth) m = fmaxf(m, fabsf(Zf[e]));
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((tid & 31) == 0) red[tid >> 5] = m;
  __syncthreads();
  m = 0.0f;
  for (int w = 0; w < nth / 32; ++w) m = fmaxf(m, red[w]);
  const bool wide = a.dtype == GEAR_F32 || a.ch;   // the rebuilding pass: bf16 hi + lo, unscaled
  int sh = 0;
  if (!wide && m > 0.0f) sh = min(max(((__float_as_int(m) >> 23) & 0xFF) - 127 - 3, -100), 100);
  const float down = __int_as_float((127 - sh) << 23), up = __int_as_float((127 + sh) << 23);
  uint8_t* img = slab + kSlabImg;
  // X Z (or R Z) operand: 16 rows of 128 channels per part, natural order
  const int parts = wide ? 2 : (a.dtype == GEAR_F16 ? 2 : 3);
  for (int e = tid; e < 16 * 128; e += nth) {
    const int n = e >> 7, c = e & 127;
    float rest = Zf[c * 16 + n] * down;
    for (int part = 0; part < parts; ++part) {
      uint16_t bitsv;
      if (a.dtype == GEAR_F16 && !wide) {
        const __half hv = __float2half_rn(rest);
        bitsv = __half_as_ushort(hv);
        rest -= __half2float(hv);
      } else {
        const __nv_bfloat16 bv = __float2bfloat16_rn(rest);
        bitsv = __bfloat16_as_ushort(bv);
        rest -= __bfloat162float(bv);
      }
      *reinterpret_cast<uint16_t*>(img + part * 4096 + zimg_offset(16, n, c)) = bitsv;
    }
  }
  if (wide) return;
  // C Z operand: zero, then each channel's ranks into its group's column block
  const int G = a.G, RB = a.r_max <= 8 ? 8 : 16, NC = G * RB > 16 ? G * RB : 16;
  const int lg = a.g == 32 ? 5 : (a.g == 64 ? 6 : 7);
  uint8_t* zc = img + parts * 4096;
  for (int e = tid; e < NC * 256 * 2 / 16; e += nth) reinterpret_cast<uint4*>(zc)[e] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  for (int e = tid; e < 128 * 16; e += nth) {
    const int c = e >> 4, j = e & 15;
    float v = 0.0f;
    if (j < RB) {
      const float z = Zf[c * 16 + j] * down;
      const __half hi = __float2half_rn(z);
      const __half lo = __float2half_rn(z - __half2float(hi));
      int m2, el;
      spread_position(a.bits, c, m2, el);
      const int n = (c >> lg) * RB + j;
      const int off = (m2 >> 3) * (NC * 128) + n * 128 + (((m2 & 7) ^ (n & 7)) << 4) + 2 * el;
      *reinterpret_cast<__half*>(zc + off) = hi;
      *reinterpret_cast<__half*>(zc + NC * 256 + off) = lo;
      v = __half2float(hi) + __half2float(lo);
    }
    Vf[e] = v;
  }
  __syncthreads();
  float* Sg = reinterpret_cast<float*>(slab + kSlabS);
  if (tid < 64) {   // S_g[j]: the group's channels in order
    const int g = tid >> 4, j = tid & 15;
    float sum = 0.0f;
    if (g < G)
      for (int c = g << lg; c < (g + 1) << lg; ++c) sum += Vf[c * 16 + j];
    Sg[tid] = sum;
  }
  if (tid == 0) {
    Sg[64] = down;
    Sg[65] = up;
    Sg[66] = 0.0f;
    Sg[67] = 0.0f;
  }
}

template <int RM, int NT>
__global__ void __launch_bounds__(NT, 512 / NT) encode_power(const EncodeArgs a) {
  constexpr int kE2Threads = NT;
  constexpr int kE2Parts = NT / 128;   // threads per row of W = M Q
  extern __shared__ __align__(128) uint8_t sm2raw[];
  E2Smem<RM, NT>& S = *reinterpret_cast<E2Smem<RM, NT>*>(sm2raw);
  const int u = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = a.r;
  const int64_t total = a.total_tiles, grid = a.grid_e1;
  const int64_t c0 = seg_first_cta((int64_t)u * a.tpu, grid, total);
  const int64_t c1 = seg_first_cta((int64_t)u * a.tpu + a.tpu - 1, grid, total);
  const int nseg = (int)(c1 - c0 + 1);
  const float* part = a.gram + (int64_t)u * a.maxc * 16384;

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
  // M = the partials summed in segment order; each thread owns the same 16
  // float4 slots of every partial, so no barrier is needed between partials
  for (int sg = 0; sg < nseg; ++sg) {
    const float4* src = reinterpret_cast<const float4*>(part + (int64_t)sg * 16384);
    float4 v[4096 / kE2Threads];
#pragma unroll
    for (int m = 0; m < 4096 / kE2Threads; ++m) v[m] = __ldcs(src + tid + m * kE2Threads);
#pragma unroll
    for (int m = 0; m < 4096 / kE2Threads; ++m) {
      const int e4 = tid + m * kE2Threads;
      float4* dst = reinterpret_cast<float4*>(&S.M[(e4 >> 5) * kMStride + ((e4 & 31) << 2)]);   // 16-byte aligned rows
      if (sg == 0) {
        *dst = v[m];
      } else {
        const float4 o = *dst;
        *dst = make_float4(o.x + v[m].x, o.y + v[m].y, o.z + v[m].z, o.w + v[m].w);
      }
    }
  }
  __syncthreads();
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
      for (int j = 0; j < RM; ++j) S.it.Wp[(wpart * 128 + i) * RM + j] = w[j];
    }
    __syncthreads();
    // G = Q^T W (upper triangle), reduced by warp then across warps
    if (tid < 128) {
      double w[RM], qv[RM];
#pragma unroll
      for (int j = 0; j < RM; ++j) {
        double v = S.it.Wp[i * RM + j];
#pragma unroll
        for (int pp = 1; pp < kE2Parts; ++pp) v += S.it.Wp[(pp * 128 + i) * RM + j];
        w[j] = v;
        qv[j] = S.Q[i * RM + j];
      }
#pragma unroll
      for (int j = 0; j < RM; ++j) S.it.Wp[i * RM + j] = w[j];
#pragma unroll
      for (int p = 0; p < RM; ++p)
#pragma unroll
        for (int q = p; q < RM; ++q) {
          double v = qv[p] * w[q];
          for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
          if (lane == 0) S.it.red[(warp * RM + p) * RM + q] = v;
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
          if (p <= q) g = S.it.red[p * RM + q] + S.it.red[(RM + p) * RM + q] + S.it.red[(2 * RM + p) * RM + q] +
                          S.it.red[(3 * RM + p) * RM + q];
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
        for (int q = 0; q < RM; ++q) S.it.Xi[p * RM + q] = X[p][q];
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
          sq = fma(S.Q[i * RM + m2], S.it.Xi[m2 * RM + j], sq);
          swv = fma(S.it.Wp[i * RM + m2], S.it.Xi[m2 * RM + j], swv);
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
        // Z rows (scaled 2^e, 16 ranks, j >= r zero) kept for the slab below;
        // M is not read again in this step
        float* Zf = S.M;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float z = 0.0f;
#pragma unroll
          for (int jj = 0; jj < RM; ++jj)
            if (jj == j && jj < r) z = (float)(zq[jj] * sL);
          Zf[i * 16 + j] = z;
        }
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
  write_z_slab(a, u, S.M, S.M + 2048);
}

// ================================================================ E3 ======
// L rows, L = R Z for every token of the block, on the tensor cores. One CTA
// per 128-token tile, two threads per token (one per 64 channels). The tile's
// input rows (E1's tensor map: 128-byte swizzled boxes), code rows
// (16-byte-chunk swizzle) and meta rows (G >= 2) arrive by tensor copies on one
// mbarrier; the unit's Z rows (E2, fp32) are read from global memory while
// they are in flight and turned into 16-bit operand images.
//
// 16-bit inputs never rebuild R. With D^ = code * scale + zero per group and
// R = X - D^ outside the outlier slots (0 there, where the code is 0):
//   L = X Z - sum_g scale_g (C Z)_g - sum_g zero_g S_g - sum_o (x_o - zero_g(o)) Z[c_o]
// with C the codes, (C Z)_g the product over the channels of group g and S_g
// the sum of Z's rows over group g. X Z takes the input tile as it landed (A
// operand, K-major) against Z split into 16-bit parts; C Z takes the codes
// spread into fp16 lanes as 1024 + code (one logic operation per pair; the
// channel order inside each 16-byte chunk is whatever the spread produces, and
// Z's block-diagonal image follows the same order) against Z split into fp16
// hi + lo, one column block per group. Z is scaled by a power of two so that the fp16 parts stay
// in range; the epilogue undoes it exactly. The thread then adds its token's
// terms: G + 2 products per rank and k outlier corrections.
//
// fp32 inputs rebuild R = x - fma(code, scale, zero) per channel (bit-identical
// to E1's residual, outlier slots 0), split as bf16 hi + lo in E1's residual
// layout, and take R Z as hi Zhi + hi Zlo + lo Zhi.
constexpr int kE3Threads = 256;   // two threads per token, one per 64-channel box

struct E3Maps {
  // per tensor: input rows, cache code rows, cache meta rows (G >= 2)
  CUtensorMap x[kMaxBatch], codes[kMaxBatch], meta[kMaxBatch];
};

template <int R>
__device__ __forceinline__ int swz_rows(int t) {   // chunk swizzle of R-byte rows (R = 32, 64, 128)
  return ((t * R) >> 7) & (R / 16 - 1);
}

// Spreads the codes of 32 channels (BITS words) into 4 chunks of eight fp16
// values, in spread_channel order: each pair is masked into the mantissas of
// 1024 (one logic operation) and 1024 is subtracted again (exact), so that the
// products carry no offset (the tensor cores' accumulation error scales with
// the largest product).
template <int BITS>
__device__ __forceinline__ void spread_codes(const uint32_t (&cw)[BITS], uint4 (&ch)[4]) {
  uint32_t u[16];
  if constexpr (BITS == 4) {
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
      for (int i = 0; i < 4; ++i) u[4 * w + i] = ((cw[w] >> (4 * i)) & 0x000F000Fu) | 0x64006400u;
  } else if constexpr (BITS == 2) {
#pragma unroll
    for (int w = 0; w < 2; ++w)
#pragma unroll
      for (int i = 0; i < 8; ++i) u[8 * w + i] = ((cw[w] >> (2 * i)) & 0x00030003u) | 0x64006400u;
  } else {
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      u[2 * w] = (cw[w] & 0x00FF00FFu) | 0x64006400u;
      u[2 * w + 1] = ((cw[w] >> 8) & 0x00FF00FFu) | 0x64006400u;
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    __half2 v = *reinterpret_cast<__half2*>(&u[i]);
    v = __hsub2(v, __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400)));
    u[i] = *reinterpret_cast<uint32_t*>(&v);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) ch[j] = make_uint4(u[4 * j], u[4 * j + 1], u[4 * j + 2], u[4 * j + 3]);
}

// Shared memory of the 16-bit E3 (from a 1024-byte-aligned base). RB columns
// per group (8 when r <= 8, else 16), NC = max(16, G * RB) columns of C Z.
template <typename T, int BITS, int RB>
struct E3ACfg {
  static constexpr int kParts = std::is_same<T, __half>::value ? 2 : 3;   // X Z: fp16 hi + lo, bf16 hi + mid + lo
  static constexpr int kX = 0;                         // input tile, then the spread codes, 32 KB
  static constexpr int kRow = 16 * BITS;               // code bytes per token
  static constexpr int kCodes = 32768;                 // code tile
  static constexpr int kMeta = kCodes + kTile * kRow;  // meta tile (G <= 4)
  static constexpr int kZx = (kMeta + kTile * 32 + 1023) & ~1023;   // X Z operand: kParts x 4 KB
  static constexpr int kZc = kZx + kParts * 4096;      // C Z operand: 2 parts x NC x 256 B
  // then, at kZc + 2 NC 256: S_g [4][16] floats with the scale and its inverse
  // (1 KB), the fp32 Z rows [128][16] (8 KB) and the barriers
  static __host__ __device__ constexpr int s_off(int NC) { return kZc + 2 * NC * 256; }
  static __host__ __device__ constexpr int zr_off(int NC) { return s_off(NC) + 1024; }
  static __host__ __device__ constexpr int bar_off(int NC) { return zr_off(NC) + 8192; }
  static __host__ __device__ constexpr int smem(int NC) { return bar_off(NC) + 64 + 1024; }   // + alignment slack
  // three barriers (24 bytes), the tensor-memory slot at +32
};

template <typename T, int BITS, int RB>
__global__ void __launch_bounds__(kE3Threads, 3) encode_lowrank_alg(const __grid_constant__ E3Maps maps,
                                                                     const EncodeArgs a) {
  using C = E1Cfg<T>;
  using F = E3ACfg<T, BITS, RB>;
  using P = typename std::conditional<std::is_same<T, __half>::value, __half, __nv_bfloat16>::type;
  extern __shared__ uint8_t e3raw[];
  uint8_t* sm = align_smem_1024(e3raw);
  uint8_t* xs = sm + F::kX;
  uint8_t* cps = xs;   // the spread codes overwrite the input tile once X Z is done
  uint8_t* cs = sm + F::kCodes;
  uint8_t* ms = sm + F::kMeta;
  uint8_t* zx = sm + F::kZx;
  uint8_t* zc = sm + F::kZc;
  const int G = a.G, k = a.k;
  const int NC = G * RB > 16 ? G * RB : 16;
  float* S = reinterpret_cast<float*>(sm + F::s_off(NC));
  const float* zr = reinterpret_cast<const float*>(sm + F::zr_off(NC));
  // [0] tile landed (one phase per tile), [1] products done (two phases per tile), [2] unit operands landed
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + F::bar_off(NC));
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + F::bar_off(NC) + 32);
  const int tid = threadIdx.x, t = tid & 127, h = tid >> 7, warp = tid >> 5;
  const int u = blockIdx.y;
  const int tile0 = blockIdx.x * a.e3_tpc;
  const int ntile = min(a.e3_tpc, a.tpu - tile0);
  const int mrb = meta_row_bytes(G, a.meta_f16);
  const bool meta_tma = mrb >= 16;
  const int lg = a.g == 32 ? 5 : (a.g == 64 ? 6 : 7);
  const int tn = u / a.Uper, ul = u % a.Uper;
  const EncodeTensor& ten = a.ten[tn];
  const uint8_t* slab = reinterpret_cast<const uint8_t*>(a.zbuf) + (int64_t)u * kZSlab;
  const uint32_t img_bytes = (uint32_t)(F::kParts * 4096 + 2 * NC * 256);
  const uint32_t tile_bytes = (uint32_t)(32768 + kTile * F::kRow + (meta_tma ? kTile * mrb : 0));
  // the tile's input rows, code rows and meta rows (one phase of bars[0])
  auto issue_tile = [&](int it) {
    const int tt0 = (tile0 + it) * kTile;
    const int crow = ul * a.n_max + a.t_off + tt0;
    mbar_arrive_expect_tx(&bars[0], tile_bytes);
    for (int b = 0; b < C::kBoxes; ++b)
      tma_load_2d(xs + b * 16384, &maps.x[tn], &bars[0], b * C::kBoxCols, ul * a.n + tt0);
    tma_load_2d(cs, &maps.codes[tn], &bars[0], 0, crow);
    if (meta_tma) tma_load_2d(ms, &maps.meta[tn], &bars[0], 0, crow);
  };
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init(&bars[2], 1);
    fence_mbarrier_init();
    // the unit's operand images, S_g and fp32 Z rows, written by E2
    mbar_arrive_expect_tx(&bars[2], img_bytes + (uint32_t)kSlabSBytes + 8192u);
    bulk_load(zx, slab + kSlabImg, img_bytes, &bars[2]);
    bulk_load(S, slab + kSlabS, (uint32_t)kSlabSBytes, &bars[2]);
    bulk_load(sm + F::zr_off(NC), slab + kSlabRows, 8192u, &bars[2]);
    issue_tile(0);
  }
  if (warp == 0) tmem_alloc(tslot, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  bool ok = __syncthreads_and(mbar_wait(&bars[2], 0));
  const float down = S[64], up = S[65];   // the images' power-of-two scale and its inverse
  int issued = 1;                          // tiles whose loads were issued
  for (int it = 0; it < ntile && ok; ++it) {
    const int t0 = (tile0 + it) * kTile;
    const bool valid = t0 + t < a.n;
    const size_t row = (size_t)(ul * a.n_max + a.t_off + t0) + t;
    // this token's outliers (channel, value) and short meta rows, fetched while the tile is in flight
    constexpr int kOF = 8;
    int oc[kOF];
    float ov[kOF];
    float2 sz[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                    make_float2(0.0f, 0.0f)};
    if (h == 0) {
#pragma unroll
      for (int i = 0; i < kOF; ++i) {
        const bool on = valid && i < k;
        oc[i] = on ? ten.oidx[row * k + i] : 0;
        ov[i] = on ? Elem16<T>::lo(reinterpret_cast<const uint16_t*>(ten.oval)[row * k + i]) : 0.0f;
      }
    }
    if (!meta_tma && valid && 8 * h < a.r_max) {   // both halves write ranks when r > 8
      if (a.meta_f16) {
        const __half2* mh = reinterpret_cast<const __half2*>(ten.meta) + row * G;
        sz[0] = __half22float2(mh[0]);
        if (G == 2) sz[1] = __half22float2(mh[1]);
      } else {
        sz[0] = reinterpret_cast<const float2*>(ten.meta)[row];
      }
    }
    ok = __syncthreads_and(mbar_wait(&bars[0], it & 1));
    if (!ok) break;
    // ---- X Z into columns [0, 16): the input tile against the parts of Z along K
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t kIdX = idesc_f16(128, 16, std::is_same<P, __nv_bfloat16>::value, false, false);
      const uint32_t xa = smem_u32(xs), za = smem_u32(zx);
      int m = 0;
#pragma unroll
      for (int part = 0; part < F::kParts; ++part)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk, ++m) {
          const uint64_t ad = smem_desc_sw128(xa + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(za + part * 4096 + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024);
          tc_mma_f16(tmem, ad, bd, kIdX, m == 0 ? 0u : 1u);
        }
      tc_commit(&bars[1]);
    }
    // ---- the meta of the token's groups into registers (the tile's meta rows
    // are overwritten by the next tile's loads before the epilogue ends)
    if (meta_tma && valid && 8 * h < a.r_max) {
      const uint8_t* mrow = ms + t * mrb;
      const int mx = mrb == 32 ? ((t >> 2) & 1) << 4 : 0;
#pragma unroll
      for (int gi = 0; gi < 4; ++gi)
        if (gi < G)
          sz[gi] = a.meta_f16 ? __half22float2(*reinterpret_cast<const __half2*>(mrow + 4 * gi))
                              : *reinterpret_cast<const float2*>(mrow + ((gi << 3) ^ mx));
    }
    // ---- spread codes of this half row, written over the input tile once X Z has read it
    const bool xz_done = mbar_wait(&bars[1], 0);
    if (!xz_done) mbar_wait(&bars[1], 0);   // nothing may overwrite the tile while the product reads it
    tc_fence_after();
    {
      const uint8_t* rowp = cs + t * F::kRow;
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int q = 2 * h + qq;   // 32-channel block
        uint32_t cw[BITS];
        if constexpr (BITS == 2) {
          const uint2 v =
              *reinterpret_cast<const uint2*>(rowp + ((((q >> 1) ^ swz_rows<F::kRow>(t)) << 4) | ((q & 1) << 3)));
          cw[0] = v.x; cw[1] = v.y;
        } else {
#pragma unroll
          for (int hh = 0; hh < BITS / 4; ++hh) {
            const uint4 v =
                *reinterpret_cast<const uint4*>(rowp + (((BITS / 4 * q + hh) ^ swz_rows<F::kRow>(t)) << 4));
            cw[4 * hh] = v.x; cw[4 * hh + 1] = v.y; cw[4 * hh + 2] = v.z; cw[4 * hh + 3] = v.w;
          }
        }
        uint4 ch[4];
        spread_codes<BITS>(cw, ch);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int m = 4 * q + j;   // chunk 0..15
          *reinterpret_cast<uint4*>(cps + (m >> 3) * 16384 + swz(t, m & 7)) = ch[j];
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(xz_done);
    tc_fence_after();
    if (ok && tid == 0) {
      // C Z into columns [32, 32 + NC): hi then lo part of Z
      const uint32_t kIdC = idesc_f16(128, NC, false, false, false);
      const uint32_t ca = smem_u32(cps), zb = smem_u32(zc);
      int m = 0;
#pragma unroll
      for (int part = 0; part < 2; ++part)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk, ++m) {
          const uint64_t ad = smem_desc_sw128(ca + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd =
              smem_desc_sw128(zb + part * NC * 256 + (kk >> 2) * (NC * 128) + (kk & 3) * 32, 16, 1024);
          tc_mma_f16(tmem + 32, ad, bd, kIdC, m == 0 ? 0u : 1u);
        }
      tc_commit(&bars[1]);
    }
    if (!ok) break;
    bool done = mbar_wait(&bars[1], 1);
    if (!done) mbar_wait(&bars[1], 1);   // the products must finish before their buffers are reused
    ok = __syncthreads_and(done);
    if (!ok) break;
    tc_fence_after();
    // the tile's shared buffers are free: the next tile loads during this epilogue
    if (tid == 0 && it + 1 < ntile) {
      issue_tile(it + 1);
      ++issued;
    }
    // ---- epilogue: thread (t, h) writes ranks [8 h, 8 h + 8) of token t
    if (8 * h < a.r_max) {
      const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
      uint32_t vx[8], vc[4][8];
      tmem_ld_32x32b_x8(lane_base + 8 * h, vx);
#pragma unroll
      for (int gi = 0; gi < 4; ++gi)
        if (gi < G) tmem_ld_32x32b_x8(lane_base + 32 + gi * RB + (RB == 16 ? 8 * h : 0), vc[gi]);
      tmem_ld_wait();
      float acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = __uint_as_float(vx[j]);
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) {
        if (gi >= G) break;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          acc[j] -= fmaf(sz[gi].x, __uint_as_float(vc[gi][j]), sz[gi].y * S[gi * 16 + 8 * h + j]);
      }
      if (valid) {
        // outlier slots: take (x_o - zero) Z[c_o] back out (their residual is 0)
        auto fix = [&](int c, float xo) {
          float zero_o = 0.0f;
#pragma unroll
          for (int gi = 0; gi < 4; ++gi)
            if (gi == (c >> lg)) zero_o = sz[gi].y;
          const float d = (xo - zero_o) * down;
          const float4 z0 = *reinterpret_cast<const float4*>(zr + c * 16 + 8 * h);
          const float4 z1 = *reinterpret_cast<const float4*>(zr + c * 16 + 8 * h + 4);
          acc[0] -= d * z0.x; acc[1] -= d * z0.y; acc[2] -= d * z0.z; acc[3] -= d * z0.w;
          acc[4] -= d * z1.x; acc[5] -= d * z1.y; acc[6] -= d * z1.z; acc[7] -= d * z1.w;
        };
        if (h == 0) {
#pragma unroll
          for (int i = 0; i < kOF; ++i)
            if (i < k) fix(oc[i], ov[i]);
        }
        for (int i = (h == 0 ? kOF : 0); i < k; ++i)
          fix(ten.oidx[row * k + i], Elem16<T>::lo(reinterpret_cast<const uint16_t*>(ten.oval)[row * k + i]));
        const int q1 = min(a.r_max, 8 * h + 8);
        if (q1 - 8 * h == 8 && (a.r_max & 7) == 0) {   // a whole 16-byte row piece
          uint32_t w[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const __half2 v2 = __floats2half2_rn(acc[2 * j] * up, acc[2 * j + 1] * up);
            w[j] = *reinterpret_cast<const uint32_t*>(&v2);
          }
          *reinterpret_cast<uint4*>(reinterpret_cast<__half*>(ten.lfac) + row * a.r_max + 8 * h) =
              make_uint4(w[0], w[1], w[2], w[3]);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (8 * h + j < q1)
              reinterpret_cast<__half*>(ten.lfac)[row * a.r_max + 8 * h + j] = __float2half_rn(acc[j] * up);
        }
      }
    }
    tc_fence_before();
    __syncthreads();   // tensor memory read before the next tile's products overwrite it
    tc_fence_after();
  }
  if (!ok && tid == 0) {
    // a bounded wait gave up (error word set): let the copies still in flight land
    mbar_wait(&bars[2], 0);
    mbar_wait(&bars[0], (issued - 1) & 1);   // every earlier tile load was waited for
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// fp32 inputs, and keys with per-channel groups (CH): rebuild R and take R Z
// as hi Zhi + hi Zlo + lo Zhi. With CH the tile's token groups' per-channel
// (scale, zero) arrive by one bulk copy of their slots (1 KB each).
template <typename T, int BITS>
struct E3Cfg {
  static constexpr int kXB = kTile * 128 * (int)sizeof(T);   // input tile (128-byte boxes)
  static constexpr int kRB = kTile * 128 * 2;          // one bf16 residual image
  static constexpr int kRow = 16 * BITS;               // code bytes per token
  static constexpr int kCB = kTile * kRow;             // code tile
  static constexpr int kMB = kTile * 32;               // meta tile (G <= 4)
  static constexpr int kX = 0;
  static constexpr int kRhi = kXB;
  static constexpr int kRlo = kRhi + kRB;
  static constexpr int kC = kRlo + kRB;
  static constexpr int kM = kC + kCB;
  static constexpr int kZ = (kM + kMB + 1023) & ~1023;   // Z image: bf16 hi | lo, 16 rows each
  static constexpr int kBar = kZ + 8192;
  static constexpr int kSmem = kBar + 64 + 1024;
};

template <typename T, int BITS, bool CH>
__global__ void __launch_bounds__(kE3Threads, 1) encode_lowrank_rebuild(const __grid_constant__ E3Maps maps,
                                                                        const EncodeArgs a) {
  using C = E1Cfg<T>;
  using F = E3Cfg<T, BITS>;
  constexpr int kPerByte = 8 / BITS;
  extern __shared__ uint8_t e3raw[];
  uint8_t* sm = align_smem_1024(e3raw);
  uint8_t* xs = sm + F::kX;
  uint8_t* rhi = sm + F::kRhi;
  uint8_t* rlo = sm + F::kRlo;
  uint8_t* cs = sm + F::kC;
  uint8_t* ms = sm + F::kM;
  uint8_t* zs = sm + F::kZ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + F::kBar);   // [0] tile landed, [1] product done
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + F::kBar + 16);
  const int tid = threadIdx.x, t = tid & 127, h = tid >> 7, warp = tid >> 5;
  const int u = blockIdx.y, t0 = blockIdx.x * kTile;
  const int G = a.G, k = a.k;
  const int mrb = meta_row_bytes(G, a.meta_f16);
  const bool meta_tma = mrb >= 16;
  const int lg = a.g == 32 ? 5 : (a.g == 64 ? 6 : 7);
  const int tn = u / a.Uper, ul = u % a.Uper;
  const EncodeTensor& ten = a.ten[tn];
  const int crow = ul * a.n_max + a.t_off + t0;
  const uint8_t* slab = reinterpret_cast<const uint8_t*>(a.zbuf) + (int64_t)u * kZSlab;
  // CH: the slots of the tile's token groups (those past the cache's slots hold no token of the tile)
  const int slot_t = a.slot0 + t0 / a.g;
  const int ngt = CH ? min(kTile / a.g, a.ch_slots - slot_t) : 0;
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbarrier_init();
    const uint32_t mbytes = CH ? (uint32_t)ngt * 1024u : (meta_tma ? (uint32_t)(kTile * mrb) : 0u);
    mbar_arrive_expect_tx(&bars[0], (uint32_t)(F::kXB + F::kCB + 8192) + mbytes);
    for (int b = 0; b < C::kBoxes; ++b)
      tma_load_2d(xs + b * 16384, &maps.x[tn], &bars[0], b * C::kBoxCols, ul * a.n + t0);
    tma_load_2d(cs, &maps.codes[tn], &bars[0], 0, crow);
    if (CH) bulk_load(ms, ten.meta + ((size_t)ul * a.ch_slots + slot_t) * 256, mbytes, &bars[0]);
    else if (meta_tma) tma_load_2d(ms, &maps.meta[tn], &bars[0], 0, crow);
    bulk_load(zs, slab + kSlabImg, 8192u, &bars[0]);   // Z image, bf16 hi | lo (E2)
  }
  if (warp == 0) tmem_alloc(tslot, 32);
  const bool valid = t0 + t < a.n;
  const size_t row = (size_t)crow + t;
  float2 szr[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
  if (!CH && !meta_tma && valid) szr[0] = reinterpret_cast<const float2*>(ten.meta)[row];
  constexpr int kOF = 8;
  int oc[kOF];
#pragma unroll
  for (int i = 0; i < kOF; ++i) oc[i] = (valid && i < k) ? ten.oidx[row * k + i] : -1;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  bool ok = mbar_wait(&bars[0], 0);
  ok = __syncthreads_and(ok);
  if (!ok && tid == 0) mbar_wait(&bars[0], 0);   // let copies still in flight land before the CTA ends

  if (ok && valid) {
    const uint8_t* mrow = ms + t * mrb;
    const int mx = mrb == 32 ? ((t >> 2) & 1) << 4 : 0;
    auto group = [&](int gi) -> float2 {
      if (!meta_tma) return gi == 0 ? szr[0] : szr[1];
      if (a.meta_f16) return __half22float2(*reinterpret_cast<const __half2*>(mrow + 4 * gi));
      return *reinterpret_cast<const float2*>(mrow + ((gi << 3) ^ mx));
    };
    // CH: (scale, zero) of channel c in the token's group
    const float2* cmeta = reinterpret_cast<const float2*>(ms) + (t / a.g) * 128;
    bool big = false;
    if (CH) {
      for (int c = 64 * h; c < 64 * h + 64; ++c) big |= !(cmeta[c].x <= 0x1p100f);
    } else {
      for (int gi = 0; gi < G; ++gi) big |= !(group(gi).x <= 0x1p100f);
    }
    auto codes32 = [&](int q, uint32_t (&cw)[BITS]) {
      const uint8_t* rowp = cs + t * F::kRow;
      if constexpr (BITS == 2) {
        const uint2 v =
            *reinterpret_cast<const uint2*>(rowp + ((((q >> 1) ^ swz_rows<F::kRow>(t)) << 4) | ((q & 1) << 3)));
        cw[0] = v.x; cw[1] = v.y;
      } else {
#pragma unroll
        for (int hh = 0; hh < BITS / 4; ++hh) {
          const uint4 v = *reinterpret_cast<const uint4*>(rowp + (((BITS / 4 * q + hh) ^ swz_rows<F::kRow>(t)) << 4));
          cw[4 * hh] = v.x; cw[4 * hh + 1] = v.y; cw[4 * hh + 2] = v.z; cw[4 * hh + 3] = v.w;
        }
      }
    };
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
    auto put = [&](int jb, const float (&rr)[8]) {
      uint32_t h4[4], l4[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const __nv_bfloat162 hb = __floats2bfloat162_rn(rr[2 * p], rr[2 * p + 1]);
        const uint32_t hbits = *reinterpret_cast<const uint32_t*>(&hb);
        const uint64_t hv = f2_pack(__uint_as_float(hbits << 16), __uint_as_float(hbits & 0xFFFF0000u));
        const uint64_t lv = f2_sub(f2_pack(rr[2 * p], rr[2 * p + 1]), hv);
        const __nv_bfloat162 lb = __floats2bfloat162_rn(f2_lo(lv), f2_hi(lv));
        h4[p] = hbits;
        l4[p] = *reinterpret_cast<const uint32_t*>(&lb);
      }
      const uint32_t off = (uint32_t)((jb >> 3) * 16384) + swz(t, jb & 7);
      *reinterpret_cast<uint4*>(rhi + off) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
      *reinterpret_cast<uint4*>(rlo + off) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
    };
    const uint32_t one = a.one_bits;
    const uint64_t one2 = f2_pack(1.0f, 1.0f);
    constexpr int kCpw = 32 / BITS;
#pragma unroll 1
    for (int q = 2 * h; q < 2 * h + 2; ++q) {   // 32 channels per pass, one group (g >= 32)
      uint32_t cw[BITS];
      codes32(q, cw);
      const float2 sz = CH ? make_float2(0.0f, 0.0f) : group((32 * q) >> lg);
      uint64_t sc2 = f2_pack(sz.x, sz.x), zr2 = f2_pack(sz.y, sz.y);
#pragma unroll
      for (int bq = 0; bq < 4; ++bq) {
        const int jb = 4 * q + bq;
        float xv[8], rr[8];
        xblock(jb, xv);
        if (!big) {
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
            const int cl = 2 * p;
            if (CH) {   // per-channel (scale, zero) of the pair
              const float2 m0 = cmeta[8 * jb + cl], m1 = cmeta[8 * jb + cl + 1];
              sc2 = f2_pack(m0.x, m1.x);
              zr2 = f2_pack(m0.y, m1.y);
            }
            const uint64_t w2 = f2_pack((float)(1 << (8 - (cl % kPerByte) * BITS)),
                                        (float)(1 << (8 - ((cl + 1) % kPerByte) * BITS)));
            const uint64_t cf = f2_sub(f2_pack(f[cl], f[cl + 1]), one2);
            const uint64_t dh = f2_fma(cf, f2_mul(sc2, w2), zr2);
            const uint64_t rv = f2_sub(f2_pack(xv[cl], xv[cl + 1]), dh);
            rr[cl] = f2_lo(rv);
            rr[cl + 1] = f2_hi(rv);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int c = 8 * bq + e;
            const float code = (float)((cw[c / kCpw] >> (BITS * (c % kCpw))) & ((1u << BITS) - 1u));
            const float2 m = CH ? cmeta[32 * q + c] : sz;
            rr[e] = __fsub_rn(xv[e], __fmaf_rn(code, m.x, m.y));
          }
        }
        put(jb, rr);
      }
    }
    for (int i = 0; i < k; ++i) {   // outlier slots of this half: residual 0
      int c = 0;
      if (i < kOF) {
#pragma unroll
        for (int i2 = 0; i2 < kOF; ++i2)
          if (i2 == i) c = oc[i2];
      } else {
        c = ten.oidx[row * k + i];
      }
      if ((c >> 6) != h) continue;
      const uint32_t off = (uint32_t)(h * 16384) + swz(t, (c & 63) >> 3) + (c & 7) * 2;
      *reinterpret_cast<uint16_t*>(rhi + off) = 0;
      *reinterpret_cast<uint16_t*>(rlo + off) = 0;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (ok && tid == 0) {
    constexpr uint32_t kIdesc = idesc_f16(128, 16, true, false, false);
    const uint32_t ah = smem_u32(rhi), al = smem_u32(rlo), zb = smem_u32(zs);
    int m = 0;
#pragma unroll
    for (int part = 0; part < 3; ++part) {   // hi Zhi, hi Zlo, lo Zhi
      const uint32_t abase = part == 2 ? al : ah;
      const uint32_t bbase = zb + (part == 1 ? 4096 : 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk, ++m) {
        const uint64_t ad = smem_desc_sw128(abase + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
        const uint64_t bd = smem_desc_sw128(bbase + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024);
        tc_mma_f16(tmem, ad, bd, kIdesc, m == 0 ? 0u : 1u);
      }
    }
    tc_commit(&bars[1]);
  }
  if (ok && 8 * h < a.r_max) {
    bool done = mbar_wait(&bars[1], 0);
    if (!done) mbar_wait(&bars[1], 0);   // the product must finish before tensor memory is freed
    tc_fence_after();
    uint32_t v[8];
    tmem_ld_32x32b_x8(tmem + ((uint32_t)((warp & 3) * 32) << 16) + 8 * h, v);
    tmem_ld_wait();
    if (valid && done) {
      const int q1 = min(a.r_max, 8 * h + 8);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (8 * h + j < q1) {
          if constexpr (sizeof(T) == 4) reinterpret_cast<float*>(ten.lfac)[row * a.r_max + 8 * h + j] = __uint_as_float(v[j]);
          else reinterpret_cast<__half*>(ten.lfac)[row * a.r_max + 8 * h + j] = __float2half_rn(__uint_as_float(v[j]));
        }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
}

// ================================================================ host =====
template <typename T, int BITS, int KMAX, bool CH>
static cudaError_t launch_e1(const XMaps& map, const EncodeArgs& a, int grid, cudaStream_t st) {
  auto kern = encode_quant_gram<T, BITS, KMAX, CH>;
  constexpr uint32_t smem = CH ? E1Cfg<T>::kSmemCh : E1Cfg<T>::kSmem;
  static std::atomic<int> smem_set[kMaxDevices];   // per device: the limit is a per-device setting
  cudaError_t e = ensure_smem_limit(kern, (int)smem, smem_set);
  if (e != cudaSuccess) return e;
  kern<<<grid, E1Cfg<T>::kThreads, smem, st>>>(map, a);
  return cudaGetLastError();
}

template <typename T, int BITS, bool CH>
static cudaError_t launch_e1_kc(const XMaps& map, const EncodeArgs& a, int grid, cudaStream_t st) {
  if (a.k == 0) return launch_e1<T, BITS, 0, CH>(map, a, grid, st);
  if (a.k == 3) return launch_e1<T, BITS, 3, CH>(map, a, grid, st);
  if (a.k <= 4) return launch_e1<T, BITS, 4, CH>(map, a, grid, st);
  if (a.k <= 8) return launch_e1<T, BITS, 8, CH>(map, a, grid, st);
  return launch_e1<T, BITS, 16, CH>(map, a, grid, st);
}

template <typename T, int BITS>
static cudaError_t launch_e1_k(const XMaps& map, const EncodeArgs& a, int grid, cudaStream_t st) {
  if constexpr (sizeof(T) == 2) {   // per-channel key groups: 16-bit caches only
    if (a.ch) return launch_e1_kc<T, BITS, true>(map, a, grid, st);
  }
  return launch_e1_kc<T, BITS, false>(map, a, grid, st);
}

template <typename T>
static cudaError_t launch_e1_b(const XMaps& map, const EncodeArgs& a, int grid, cudaStream_t st) {
  switch (a.bits) {
    case 2: return launch_e1_k<T, 2>(map, a, grid, st);
    case 4: return launch_e1_k<T, 4>(map, a, grid, st);
    default: return launch_e1_k<T, 8>(map, a, grid, st);
  }
}

template <typename T, int BITS, int RB>
static cudaError_t launch_e3a(const E3Maps& maps, const EncodeArgs& a, dim3 grid, cudaStream_t st) {
  auto kern = encode_lowrank_alg<T, BITS, RB>;
  const int smem = E3ACfg<T, BITS, RB>::smem(a.G * RB > 16 ? a.G * RB : 16);
  static std::atomic<int> smem_set[kMaxDevices];
  cudaError_t e = ensure_smem_limit(kern, smem, smem_set);
  if (e != cudaSuccess) return e;
  kern<<<grid, kE3Threads, smem, st>>>(maps, a);
  return cudaGetLastError();
}

template <typename T, int BITS, bool CH>
static cudaError_t launch_e3f(const E3Maps& maps, const EncodeArgs& a, dim3 grid, cudaStream_t st) {
  auto kern = encode_lowrank_rebuild<T, BITS, CH>;
  constexpr int smem = E3Cfg<T, BITS>::kSmem;
  static std::atomic<int> smem_set[kMaxDevices];
  cudaError_t e = ensure_smem_limit(kern, smem, smem_set);
  if (e != cudaSuccess) return e;
  kern<<<grid, kE3Threads, smem, st>>>(maps, a);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_e3_b(const E3Maps& maps, const EncodeArgs& a, cudaStream_t st) {
  dim3 grid(a.tpu, a.U);
  if constexpr (sizeof(T) == 4) {
    switch (a.bits) {
      case 2: return launch_e3f<float, 2, false>(maps, a, grid, st);
      case 4: return launch_e3f<float, 4, false>(maps, a, grid, st);
      default: return launch_e3f<float, 8, false>(maps, a, grid, st);
    }
  } else if (a.ch) {
    switch (a.bits) {
      case 2: return launch_e3f<T, 2, true>(maps, a, grid, st);
      case 4: return launch_e3f<T, 4, true>(maps, a, grid, st);
      default: return launch_e3f<T, 8, true>(maps, a, grid, st);
    }
  } else {
    grid.x = (a.tpu + a.e3_tpc - 1) / a.e3_tpc;   // e3_tpc tiles per CTA
    const bool r8 = a.r_max <= 8;
    switch (a.bits) {
      case 2: return r8 ? launch_e3a<T, 2, 8>(maps, a, grid, st) : launch_e3a<T, 2, 16>(maps, a, grid, st);
      case 4: return r8 ? launch_e3a<T, 4, 8>(maps, a, grid, st) : launch_e3a<T, 4, 16>(maps, a, grid, st);
      default: return r8 ? launch_e3a<T, 8, 8>(maps, a, grid, st) : launch_e3a<T, 8, 16>(maps, a, grid, st);
    }
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
  // E3 (16-bit inputs): consecutive tiles of one unit per CTA, so that the
  // unit's operands load once per CTA; at least two waves of three CTAs per SM
  {
    const int64_t waves2 = (int64_t)num_sms * 3 * 2;
    int64_t tpc = a.total_tiles / (waves2 > 0 ? waves2 : 1);
    a.e3_tpc = (int)(tpc < 1 ? 1 : (tpc > 8 ? 8 : tpc));
    if (a.e3_tpc > a.tpu) a.e3_tpc = a.tpu;
  }

  const int grid = a.grid_e1;
  cudaError_t e;
  if (a.dtype == GEAR_F16) e = launch_e1_b<__half>(xm, a, grid, st);
  else if (a.dtype == GEAR_BF16) e = launch_e1_b<__nv_bfloat16>(xm, a, grid, st);
  else e = launch_e1_b<float>(xm, a, grid, st);
  if (e != cudaSuccess) return e;
  if (a.r == 0) return cudaSuccess;

  {
    const int RM = a.r <= 4 ? 4 : (a.r <= 8 ? 8 : 16);
    const bool wide = a.U <= num_sms;   // one wave: 512 threads per unit
    const int ri = RM == 4 ? 0 : (RM == 8 ? 1 : 2);
    static std::atomic<int> smem_set[2][3][kMaxDevices];
    if (wide) {
      const size_t sm2 = RM == 4 ? sizeof(E2Smem<4, 512>) : (RM == 8 ? sizeof(E2Smem<8, 512>) : sizeof(E2Smem<16, 512>));
      auto kern = RM == 4 ? encode_power<4, 512> : (RM == 8 ? encode_power<8, 512> : encode_power<16, 512>);
      e = ensure_smem_limit(kern, (int)sm2, smem_set[0][ri]);
      if (e != cudaSuccess) return e;
      kern<<<a.U, 512, sm2, st>>>(a);
    } else {
      const size_t sm2 = RM == 4 ? sizeof(E2Smem<4, 256>) : (RM == 8 ? sizeof(E2Smem<8, 256>) : sizeof(E2Smem<16, 256>));
      auto kern = RM == 4 ? encode_power<4, 256> : (RM == 8 ? encode_power<8, 256> : encode_power<16, 256>);
      e = ensure_smem_limit(kern, (int)sm2, smem_set[1][ri]);
      if (e != cudaSuccess) return e;
      kern<<<a.U, 256, sm2, st>>>(a);
    }
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  if (a.dtype == GEAR_F16) return launch_e3_b<__half>(m3, a, st);
  if (a.dtype == GEAR_BF16) return launch_e3_b<__nv_bfloat16>(m3, a, st);
  return launch_e3_b<float>(m3, a, st);
}

}  // namespace gear
