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
// Split-K (flash-decoding style): kernel decode_split handles a chunk of the
// compressed tokens of one (batch, kv head) for all query heads sharing that
// kv head, keeping an online softmax; the last split of each unit handles the
// buffer. decode_combine merges the splits by log-sum-exp.
#include "common.cuh"
#include "decode.cuh"

namespace gear {

constexpr int kDThreads = 128;
constexpr int kDTile = 128;
constexpr int kMaxHq = 8;
constexpr int kMaxW = 32;      // 8-bit codes: 32 words per token
constexpr int kMaxK = 16;
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

struct DecodeSmem {
  float q[kMaxHq][128];
  float qsum[kMaxHq][4];
  float u[kMaxHq][kMaxR];          // Rf_K^T q of the current block
  float alr[kMaxHq][kMaxR];        // sum_t p_t L^V_t of the tile
  float rfk[kMaxR][128];           // Rf of the current block (K, V)
  float rfv[kMaxR][128];
  uint32_t codes[kDTile][kMaxW + 1];
  float2 meta[kDTile][4];
  uint8_t oidx[kDTile][kMaxK];
  float oval[kDTile][kMaxK];
  float lf[kDTile][kMaxR];
  float sc[kMaxHq][kDTile];        // scores, then probabilities
  float acc[kMaxHq][128];
  float m[kMaxHq], l[kMaxHq], alpha[kMaxHq];
  float red[kMaxHq][4];
};

__device__ __forceinline__ int block_of(const DecodeArgs& a, int t) {
  return t < a.blk0_len ? 0 : 1 + (t - a.blk0_len) / a.n_b;
}
__device__ __forceinline__ int block_start(const DecodeArgs& a, int b) {
  return b == 0 ? 0 : a.blk0_len + (b - 1) * a.n_b;
}
__device__ __forceinline__ int block_end(const DecodeArgs& a, int b) {
  return b == 0 ? a.blk0_len : a.blk0_len + b * a.n_b;
}

// stage tokens [t0, t0 + nt) of one compressed tensor of unit u
template <typename T>
__device__ void stage_tile(const DecodeArgs& a, const CacheView& cv, DecodeSmem& s, int u, int t0, int nt) {
  const size_t row0 = (size_t)u * a.n_max + t0;
  const int W = a.W, G = a.G, k = a.k, rm = a.r_max;
  for (int e = threadIdx.x; e < nt * W; e += kDThreads) s.codes[e / W][e % W] = cv.codes[row0 * W + e];
  for (int e = threadIdx.x; e < nt * G; e += kDThreads)
    s.meta[e / G][e % G] = reinterpret_cast<const float2*>(cv.meta)[row0 * G + e];
  for (int e = threadIdx.x; e < nt * k; e += kDThreads) {
    s.oidx[e / k][e % k] = cv.oidx[row0 * k + e];
    s.oval[e / k][e % k] = load_elem<T>(cv.oval, row0 * k + e);
  }
  for (int e = threadIdx.x; e < nt * rm; e += kDThreads) s.lf[e / rm][e % rm] = load_lfac<T>(cv.lfac, row0 * rm + e);
}

__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// online-softmax update of the tile's scores s.sc[hh][0..nt): converts them to
// probabilities relative to the new running max and sets s.alpha.
__device__ void softmax_tile(DecodeSmem& s, int hq, int nt) {
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  for (int hh = 0; hh < hq; ++hh) {
    float v = t < nt ? s.sc[hh][t] : -INFINITY;
    v = warp_max(v);
    if (lane == 0) s.red[hh][w] = v;
  }
  __syncthreads();
  for (int hh = 0; hh < hq; ++hh) {
    float tm = fmaxf(fmaxf(s.red[hh][0], s.red[hh][1]), fmaxf(s.red[hh][2], s.red[hh][3]));
    float mnew = fmaxf(s.m[hh], tm);
    float p = t < nt ? exp2f(s.sc[hh][t] - mnew) : 0.0f;
    __syncwarp();
    if (t < kDTile) s.sc[hh][t] = p;
    float ps = warp_sum(p);
    __syncthreads();
    if (lane == 0) s.red[hh][w] = ps;
    __syncthreads();
    if (t == 0) {
      float al = exp2f(s.m[hh] - mnew);
      s.alpha[hh] = al;
      s.l[hh] = s.l[hh] * al + (s.red[hh][0] + s.red[hh][1] + s.red[hh][2] + s.red[hh][3]);
      s.m[hh] = mnew;
    }
  }
  __syncthreads();
}

template <typename T, int BITS>
__global__ void __launch_bounds__(kDThreads) decode_split(const DecodeArgs a) {
  extern __shared__ uint8_t dsm_raw[];
  DecodeSmem& s = *reinterpret_cast<DecodeSmem*>(dsm_raw);
  const int unit = blockIdx.y;              // b * H + h
  const int b = unit / a.H, h = unit % a.H;
  const int split = blockIdx.x;
  const int hq = a.hq;
  const int tid = threadIdx.x;
  constexpr uint32_t kMask = (1u << BITS) - 1u;
  constexpr int kPerWord = 32 / BITS;

  // query heads j = h*hq .. h*hq + hq - 1
  for (int e = tid; e < hq * 128; e += kDThreads) {
    const int hh = e >> 7, c = e & 127;
    s.q[hh][c] = load_elem<T>(a.q, ((size_t)b * a.Hq + h * hq + hh) * 128 + c);
  }
  for (int e = tid; e < hq * 128; e += kDThreads) s.acc[e >> 7][e & 127] = 0.0f;
  if (tid < kMaxHq) { s.m[tid] = -INFINITY; s.l[tid] = 0.0f; }
  __syncthreads();
  if (tid < hq * a.G) {
    const int hh = tid / a.G, gg = tid % a.G;
    float v = 0.0f;
    for (int c = gg * a.g; c < (gg + 1) * a.g; ++c) v += s.q[hh][c];
    s.qsum[hh][gg] = v;
  }
  __syncthreads();

  if (split < a.nsplit_comp) {
    const int c0 = split * a.chunk;
    const int c1 = min(a.n_comp, c0 + a.chunk);
    int cur_blk = -1, rb = 0;
    for (int t0 = c0; t0 < c1;) {
      const int blk = block_of(a, t0);
      const int t1 = min(min(t0 + kDTile, c1), block_end(a, blk));
      const int nt = t1 - t0;
      if (blk != cur_blk) {
        cur_blk = blk;
        rb = blk == 0 ? a.blk0_rank : a.buffer_rank;
        const size_t rf0 = ((size_t)unit * a.nblk_max + blk) * a.r_max * 128;
        for (int e = tid; e < a.r_max * 128; e += kDThreads) {
          s.rfk[e >> 7][e & 127] = a.K.rfac[rf0 + e];
          s.rfv[e >> 7][e & 127] = a.V.rfac[rf0 + e];
        }
        __syncthreads();
        if (tid < hq * kMaxR) {
          const int hh = tid / kMaxR, j = tid % kMaxR;
          float v = 0.0f;
          if (j < rb)
            for (int c = 0; c < 128; ++c) v = fmaf(s.rfk[j][c], s.q[hh][c], v);
          s.u[hh][j] = v;
        }
      }
      // ---------------- keys: one thread per token
      stage_tile<T>(a, a.K, s, unit, t0, nt);
      __syncthreads();
      if (tid < nt) {
        float sc[kMaxHq];
        for (int hh = 0; hh < kMaxHq; ++hh) sc[hh] = 0.0f;
        for (int gg = 0; gg < a.G; ++gg) {
          float dot[kMaxHq];
          for (int hh = 0; hh < kMaxHq; ++hh) dot[hh] = 0.0f;
          for (int c = gg * a.g; c < (gg + 1) * a.g; ++c) {
            const uint32_t code = (s.codes[tid][c / kPerWord] >> (BITS * (c % kPerWord))) & kMask;
            const float cf = (float)code;
            for (int hh = 0; hh < hq; ++hh) dot[hh] = fmaf(cf, s.q[hh][c], dot[hh]);
          }
          const float2 sz = s.meta[tid][gg];
          for (int hh = 0; hh < hq; ++hh) sc[hh] += sz.x * dot[hh] + sz.y * s.qsum[hh][gg];
        }
        for (int j = 0; j < rb; ++j) {
          const float lj = s.lf[tid][j];
          for (int hh = 0; hh < hq; ++hh) sc[hh] = fmaf(lj, s.u[hh][j], sc[hh]);
        }
        for (int i = 0; i < a.k; ++i) {
          const int c = s.oidx[tid][i];
          float lr = 0.0f;
          for (int j = 0; j < rb; ++j) lr = fmaf(s.lf[tid][j], s.rfk[j][c], lr);
          const float fix = s.oval[tid][i] - (s.meta[tid][c / a.g].y + lr);
          for (int hh = 0; hh < hq; ++hh) sc[hh] = fmaf(s.q[hh][c], fix, sc[hh]);
        }
        for (int hh = 0; hh < hq; ++hh) s.sc[hh][tid] = sc[hh] * a.scale_log2;
      }
      __syncthreads();
      softmax_tile(s, hq, nt);
      // ---------------- values
      stage_tile<T>(a, a.V, s, unit, t0, nt);
      __syncthreads();
      {
        const int c = tid;  // one thread per channel
        const int w = c / kPerWord, sh = BITS * (c % kPerWord), gg = c / a.g;
        float acc[kMaxHq];
        for (int hh = 0; hh < kMaxHq; ++hh) acc[hh] = hh < hq ? s.acc[hh][c] * s.alpha[hh] : 0.0f;
        for (int t = 0; t < nt; ++t) {
          const uint32_t code = (s.codes[t][w] >> sh) & kMask;
          const float2 sz = s.meta[t][gg];
          const float v = __fmaf_rn((float)code, sz.x, sz.y);
          for (int hh = 0; hh < hq; ++hh) acc[hh] = fmaf(s.sc[hh][t], v, acc[hh]);
        }
        for (int hh = 0; hh < hq; ++hh) s.acc[hh][c] = acc[hh];
      }
      if (tid < hq * kMaxR) {
        const int hh = tid / kMaxR, j = tid % kMaxR;
        float v = 0.0f;
        if (j < rb)
          for (int t = 0; t < nt; ++t) v = fmaf(s.sc[hh][t], s.lf[t][j], v);
        s.alr[hh][j] = v;
      }
      __syncthreads();
      {
        const int c = tid;
        for (int hh = 0; hh < hq; ++hh) {
          float v = s.acc[hh][c];
          for (int j = 0; j < rb; ++j) v = fmaf(s.alr[hh][j], s.rfv[j][c], v);
          s.acc[hh][c] = v;
        }
      }
      __syncthreads();
      if (tid < nt) {
        for (int i = 0; i < a.k; ++i) {
          const int c = s.oidx[tid][i];
          float lr = 0.0f;
          for (int j = 0; j < rb; ++j) lr = fmaf(s.lf[tid][j], s.rfv[j][c], lr);
          const float fix = s.oval[tid][i] - (s.meta[tid][c / a.g].y + lr);
          for (int hh = 0; hh < hq; ++hh) atomicAdd(&s.acc[hh][c], s.sc[hh][tid] * fix);
        }
      }
      __syncthreads();
      t0 = t1;
    }
  } else {
    // ---------------- the streaming buffer: exact tokens
    const size_t brow = (size_t)unit * a.n_b;
    for (int t0 = 0; t0 < a.n_buf; t0 += kDTile) {
      const int nt = min(kDTile, a.n_buf - t0);
      if (tid < nt) {
        float sc[kMaxHq];
        for (int hh = 0; hh < kMaxHq; ++hh) sc[hh] = 0.0f;
        for (int c = 0; c < 128; ++c) {
          const float x = load_elem<T>(a.K.buf, (brow + t0 + tid) * 128 + c);
          for (int hh = 0; hh < hq; ++hh) sc[hh] = fmaf(x, s.q[hh][c], sc[hh]);
        }
        for (int hh = 0; hh < hq; ++hh) s.sc[hh][tid] = sc[hh] * a.scale_log2;
      }
      __syncthreads();
      softmax_tile(s, hq, nt);
      {
        const int c = tid;
        for (int hh = 0; hh < hq; ++hh) {
          float v = s.acc[hh][c] * s.alpha[hh];
          for (int t = 0; t < nt; ++t) v = fmaf(s.sc[hh][t], load_elem<T>(a.V.buf, (brow + t0 + t) * 128 + c), v);
          s.acc[hh][c] = v;
        }
      }
      __syncthreads();
    }
  }

  // ---------------- partial result of this split
  for (int hh = 0; hh < hq; ++hh) {
    float* dst = a.part + (((size_t)b * a.Hq + h * hq + hh) * a.nsplit + split) * 130;
    if (tid == 0) { dst[0] = s.m[hh]; dst[1] = s.l[hh]; }
    dst[2 + tid] = s.acc[hh][tid];
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
  int nsc = 0;
  if (a.n_comp > 0) {
    nsc = (4 * num_sms + units - 1) / units;
    int maxs = (a.n_comp + 255) / 256;
    if (nsc > maxs) nsc = maxs;
    if (nsc < 1) nsc = 1;
    a.chunk = (a.n_comp + nsc - 1) / nsc;
    nsc = (a.n_comp + a.chunk - 1) / a.chunk;
  } else {
    a.chunk = 1;
  }
  a.nsplit_comp = nsc;
  a.nsplit = nsc + (a.n_buf > 0 ? 1 : 0);
}

size_t decode_workspace_bytes(int B, int Hq, int nsplit) { return (size_t)B * Hq * nsplit * 130 * sizeof(float); }

template <typename T>
static cudaError_t launch_split(const DecodeArgs& a, cudaStream_t st) {
  dim3 grid(a.nsplit, a.B * a.H);
  const size_t smem = sizeof(DecodeSmem);
  cudaError_t e;
  switch (a.bits) {
    case 2:
      e = cudaFuncSetAttribute(decode_split<T, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      decode_split<T, 2><<<grid, kDThreads, smem, st>>>(a);
      break;
    case 4:
      e = cudaFuncSetAttribute(decode_split<T, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      decode_split<T, 4><<<grid, kDThreads, smem, st>>>(a);
      break;
    default:
      e = cudaFuncSetAttribute(decode_split<T, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      decode_split<T, 8><<<grid, kDThreads, smem, st>>>(a);
      break;
  }
  return cudaGetLastError();
}

cudaError_t decode_launch(const DecodeArgs& a, cudaStream_t st) {
  cudaError_t e;
  if (a.dtype == GEAR_F16) e = launch_split<__half>(a, st);
  else if (a.dtype == GEAR_BF16) e = launch_split<__nv_bfloat16>(a, st);
  else e = launch_split<float>(a, st);
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
