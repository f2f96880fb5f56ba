// decode.cu -- decode-step attention over a GEAR-compressed KV cache: the
// split-K combine, the launch plan and dispatch, and the dense export. The
// attention kernel itself (decode_warp) lives in decode_warp.cuh and is
// instantiated per cache dtype in decode_f16.cu, decode_bf16.cu, decode_f32.cu.
#include <string.h>
#include "common.cuh"
#include "decode.cuh"

namespace gear {

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

template <typename TO>
__global__ void __launch_bounds__(128) decode_combine(const DecodeArgs a) {
  const int bj = blockIdx.x;  // b * Hq + j
  const int c = threadIdx.x;
  const float* p = a.part + (size_t)bj * a.nsplit * 130;
  // the warps that met this query head's unit wrote partial rows 0 .. nseg-1
  int nseg = 1;
  if (a.rows && a.tot_tokens > 0) {
    // paged layout: the unit's start in the rows' token space (see decode_warp)
    const int b = bj / a.Hq, h = (bj % a.Hq) / a.hq;
    auto len_of = [&](int r) {
      const int nb = __ldg(a.rows + a.B + r);
      return nb > 0 ? __ldg(a.rows + r) + (nb - 1) * a.n_b : 0;
    };
    int64_t start = 0;
    for (int r = 0; r < b; ++r) start += (int64_t)a.H * len_of(r);
    const int len = len_of(b);
    start += (int64_t)h * len;
    nseg = len > 0 ? (int)((start + len - 1) / a.seg_tokens - start / a.seg_tokens + 1) : 0;
  } else if (a.n_comp > 0) {
    const int64_t u = (int64_t)(bj / a.Hq) * a.H + (bj % a.Hq) / a.hq, n = a.n_comp;
    nseg = (int)(((u + 1) * n - 1) / a.seg_tokens - (u * n) / a.seg_tokens + 1);
  }
  float M = -INFINITY;
  for (int s = 0; s < nseg; ++s) M = fmaxf(M, p[s * 130]);
  float den = 0.0f, num = 0.0f;
  for (int s = 0; s < nseg; ++s) {
    const float m = p[s * 130];
    if (m == -INFINITY) continue;   // a split without a finite score contributes nothing
    const float w = exp2f(m - M);
    den = fmaf(p[s * 130 + 1], w, den);
    num = fmaf(p[s * 130 + 2 + c], w, num);
  }
  const float o = den > 0.0f ? num / den : 0.0f;   // a row whose every token is padding gives 0
  TO* out = reinterpret_cast<TO*>(a.out) + (size_t)bj * 128 + c;
  if constexpr (sizeof(TO) == 4) *out = o;
  else if constexpr (std::is_same<TO, __half>::value) *out = __float2half_rn(o);
  else *out = __float2bfloat16_rn(o);
}

void decode_plan(DecodeArgs& a, int num_sms) {
  const int units = a.B * a.H;
  auto r16 = [](int x) { return (x + 15) & ~15; };
  const int esz = a.dtype == GEAR_F32 ? 4 : 2;   // oval and L rows share the width
  TileLayout& L = a.tl;
  L.cb = kDTile * a.W * 4;
  const int mrb = meta_row_bytes(a.G, a.meta_f16);
  L.mb = kDTile * mrb;
  L.oval = r16(kDTile * a.k);
  L.lf = L.oval + r16(kDTile * a.k * esz);
  L.rb = L.lf + r16(kDTile * a.r_max * esz);
  L.meta0 = 0;
  L.rest0 = L.meta0 + 4 * L.mb;
  L.floats = L.rest0 + 4 * L.rb;
  const int hq = a.hq;
  // qw, u, alr, w, accx, and with per-channel key groups qk, zk
  const int floats = hq * 128 + 2 * hq * kMaxR + kWStride * a.G * hq + hq * 128 + (a.kc ? hq * 128 + 128 : 0);
  L.bars = L.floats + r16(floats * 4);
  L.bytes = (L.bars + 16 + 255) & ~255;   // meta tiles stay 256-byte aligned
  const int nmeta = a.kc ? 1 : 2;   // per-channel key groups: no per-token key meta rows
  const int meta_tx = mrb >= 16 ? nmeta * L.mb : 0;
  L.tx_part = 2 * L.cb + meta_tx;
  L.tx_full = L.tx_part + 2 * kDTile * (a.k + a.k * esz + a.r_max * esz) + (mrb >= 16 ? 0 : nmeta * L.mb);
  // stream-K over the units' compressed tokens: one wave of resident warps,
  // each taking an equal run of tokens (a multiple of 32)
  const int smem_cta = 1024 + 16 * L.cb + 4 * L.bytes;
  const int by_smem = 233472 / (smem_cta + 1024);   // 228 KiB per SM, 1 KiB reserved per CTA
  const int by_regs = hq <= 2 ? 4 : (hq == 4 ? 2 : 1);
  const long long resident = (long long)num_sms * (by_smem < by_regs ? (by_smem > 0 ? by_smem : 1) : by_regs) * 4;
  const long long tot = a.rows ? (long long)a.tot_tokens : (long long)a.n_comp * units;
  if (tot > 0) {
    long long seg = (tot + resident - 1) / resident;
    seg = (seg + kDTile - 1) / kDTile * kDTile;
    a.seg_tokens = (int)seg;
    a.total_splits = (int)((tot + seg - 1) / seg);
    a.nsplit = (int)((a.n_comp + seg - 1) / seg) + 1;
  } else {
    a.seg_tokens = 0;
    a.total_splits = units;
    a.nsplit = 1;
  }
}

size_t decode_workspace_bytes(int B, int Hq, int nsplit) { return (size_t)B * Hq * nsplit * 130 * sizeof(float); }

cudaError_t decode_launch(const DecodeArgs& a, cudaStream_t st) {
  cudaError_t e = cudaSuccess;
  if (a.n_comp > 0 || a.n_buf > 0) {
    DecodeMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (a.n_comp > 0) {
      PFN_encodeTiled enc = tensor_map_encoder();
      if (!enc) return cudaErrorNotSupported;
      const uint64_t rows = a.table ? (uint64_t)a.num_pages * a.H * a.page_tokens : (uint64_t)a.B * a.H * a.n_max;
      bool ok = cache_row_map(enc, &maps.kc, a.K.codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.W, rows, kDTile) &&
                cache_row_map(enc, &maps.vc, a.V.codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.W, rows, kDTile);
      // meta rows of 16 bytes or more come by tensor copy, as 32-bit words
      const int mrb = meta_row_bytes(a.G, a.meta_f16);
      if (ok && mrb >= 16)
        ok = (a.kc || cache_row_map(enc, &maps.km, a.K.meta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, mrb / 4, rows, kDTile)) &&
             cache_row_map(enc, &maps.vm, a.V.meta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, mrb / 4, rows, kDTile);
      if (!ok) return cudaErrorInvalidValue;
    }
    if (a.kc) e = decode_warp_launch_kc(maps, a, st);
    else if (a.dtype == GEAR_F16) e = decode_warp_launch_f16(maps, a, st);
    else if (a.dtype == GEAR_BF16) e = decode_warp_launch_bf16(maps, a, st);
    else e = decode_warp_launch_f32(maps, a, st);
  }
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
      float2 sz;
      if (a.ch) {   // token group slot: block 0 in groups of g, then whole groups per flushed block
        const int slot = t < a.blk0_len ? t / a.g : (a.blk0_len + a.g - 1) / a.g + (t - a.blk0_len) / a.g;
        sz = reinterpret_cast<const float2*>(a.C.meta)[((size_t)u * a.ch_slots + slot) * 128 + c];
      } else {
        sz = a.meta_f16 ? __half22float2(reinterpret_cast<const __half2*>(a.C.meta)[row * a.G + c / a.g])
                        : reinterpret_cast<const float2*>(a.C.meta)[row * a.G + c / a.g];
      }
      v = __fmaf_rn((float)code, sz.x, sz.y);
      const int rp = rpad_of(a.r_max);
      const float* rf = a.C.rfac + (((size_t)u * a.nblk_max + blk) * 128 + c) * rp;
      for (int j = 0; j < rb; ++j) v = fmaf(load_lfac<T>(a.C.lfac, row * a.r_max + j), rf[j], v);
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
