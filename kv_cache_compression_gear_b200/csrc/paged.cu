// paged.cu -- kernels of the paged cache layout (host logic in api.cu).
//
// A paged cache keeps each row's compressed tokens in pool pages of P tokens:
// token t of row b, head h is pool row (table[b][t / P] * H + h) * P + t % P.
// Encodes run on a contiguous staging copy (the same encoder kernels as a
// contiguous cache); paged_scatter then moves every token row and the block's
// Rf into place. These kernels move bytes only: no arithmetic of the codec.
#include "paged.cuh"

namespace gear {

__global__ void __launch_bounds__(256) paged_set(const PagedSet s) {
  for (int i = threadIdx.x; i < s.ntab; i += blockDim.x) s.table[s.tab_idx[i]] = s.tab_val[i];
  for (int i = threadIdx.x; i < s.nrow; i += blockDim.x) {
    const int b = s.row[i];
    s.rows[b] = s.b0[i];
    s.rows[s.B + b] = s.nblk[i];
    s.rows[2 * s.B + b] = s.nbuf[i];
  }
}

// grid (n * H, 2 tensors): unit (row[i], h) of the cache buffer -> unit
// (i0 + i) * H + h of the staging input, 16 bytes per thread and step.
__global__ void __launch_bounds__(256) paged_gather(const uint4* __restrict__ sk, const uint4* __restrict__ sv,
                                                    uint4* __restrict__ dk, uint4* __restrict__ dv, int H, int wpu,
                                                    const PagedRows r) {
  const int ul = blockIdx.x, i = ul / H, h = ul % H;
  const int64_t su = (int64_t)r.row[i] * H + h, du = (int64_t)(r.i0 + i) * H + h;
  const uint4* s = blockIdx.y ? sv : sk;
  uint4* d = blockIdx.y ? dv : dk;
  for (int w = threadIdx.x; w < wpu; w += blockDim.x) d[du * wpu + w] = s[su * wpu + w];
}

// Copies nt token rows of bpr bytes: source rows srow0 .. srow0 + nt - 1,
// destination rows drow[0 .. nt). Whole 32-bit words when rows allow it.
__device__ __forceinline__ void copy_rows(uint8_t* dst, const uint8_t* src, int bpr, const int64_t* drow,
                                          int64_t srow0, int nt) {
  if (bpr <= 0) return;
  if ((bpr & 3) == 0) {
    const int wpr = bpr >> 2;
    uint32_t* d = reinterpret_cast<uint32_t*>(dst);
    const uint32_t* s = reinterpret_cast<const uint32_t*>(src);
    for (int e = threadIdx.x; e < nt * wpr; e += blockDim.x) {
      const int tok = e / wpr, w = e - tok * wpr;
      d[drow[tok] * wpr + w] = s[(srow0 + tok) * wpr + w];
    }
  } else {
    for (int e = threadIdx.x; e < nt * bpr; e += blockDim.x) {
      const int tok = e / bpr, w = e - tok * bpr;
      dst[drow[tok] * bpr + w] = src[(srow0 + tok) * bpr + w];
    }
  }
}

// grid (ceil(n / 32), r.n * H): 32 tokens of one unit per CTA; the CTAs of
// x = 0 also move the unit's Rf block.
__global__ void __launch_bounds__(128) paged_scatter(const ScatterArgs s, const PagedRows r) {
  const int ul = blockIdx.y, i = ul / s.H, h = ul % s.H;
  const int b = r.row[i];
  const int64_t su = (int64_t)(r.i0 + i) * s.H + h, du = (int64_t)b * s.H + h;
  const int tau0 = blockIdx.x * 32;
  const int nt = min(32, s.n - tau0);
  __shared__ int64_t drow[32];
  if ((int)threadIdx.x < nt) {
    const int t = r.t0[i] + tau0 + threadIdx.x;
    int pg = s.table[(int64_t)b * s.ppr + t / s.P];
    pg = min(max(pg, 0), s.num_pages - 1);   // the host maps every page a row's tokens reach
    drow[threadIdx.x] = ((int64_t)pg * s.H + h) * s.P + t % s.P;
  }
  __syncthreads();
  const int64_t srow0 = su * s.nmax_s + tau0;
  copy_rows(s.d_codes, s.s_codes, s.wb, drow, srow0, nt);
  copy_rows(s.d_meta, s.s_meta, s.mb, drow, srow0, nt);
  copy_rows(s.d_oidx, s.s_oidx, s.kb, drow, srow0, nt);
  copy_rows(s.d_oval, s.s_oval, s.ob, drow, srow0, nt);
  copy_rows(s.d_lfac, s.s_lfac, s.lb, drow, srow0, nt);
  if (blockIdx.x == 0) {
    float* d = s.d_rfac + (du * s.nblk_max + r.blk[i]) * s.rf_floats;
    const float* src = s.s_rfac + su * s.rf_floats;   // the staging copy holds one block
    for (int e = threadIdx.x; e < s.rf_floats; e += blockDim.x) d[e] = src[e];
    if (s.ch) {   // the block's token-group slots (1 KB each)
      const int nf = (s.n + s.g - 1) / s.g * 256;
      const float* ms = reinterpret_cast<const float*>(s.s_meta) + su * s.ch_slots_s * 256;
      float* md = reinterpret_cast<float*>(s.d_meta) + (du * s.ch_slots_d + r.s0[i]) * 256;
      for (int e = threadIdx.x; e < nf; e += blockDim.x) md[e] = ms[e];
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(128) paged_append(const PagedAppend a) {
  const int ul = blockIdx.x, i = ul / a.H, h = ul % a.H, c = threadIdx.x;
  const int b = a.row[i];
  const size_t dst = (((size_t)b * a.H + h) * a.n_b + a.slot[i]) * 128 + c;
  const size_t src = ((size_t)(a.i0 + i) * a.H + h) * 128 + c;
  reinterpret_cast<T*>(a.kbuf)[dst] = reinterpret_cast<const T*>(a.kn)[src];
  reinterpret_cast<T*>(a.vbuf)[dst] = reinterpret_cast<const T*>(a.vn)[src];
  if (h == 0 && c == 0) {
    a.krows[a.B + b] = a.nblk[i];
    a.krows[2 * a.B + b] = a.slot[i] + 1;
    a.vrows[a.B + b] = a.nblk[i];
    a.vrows[2 * a.B + b] = a.slot[i] + 1;
  }
}

cudaError_t paged_set_launch(const PagedSet& s, cudaStream_t st) {
  if (s.ntab == 0 && s.nrow == 0) return cudaSuccess;
  paged_set<<<1, 256, 0, st>>>(s);
  return cudaGetLastError();
}

cudaError_t paged_gather_launch(const void* sk, const void* sv, void* dk, void* dv, int H, int unit_bytes,
                                const PagedRows& r, cudaStream_t st) {
  if (r.n == 0) return cudaSuccess;
  paged_gather<<<dim3(r.n * H, 2), 256, 0, st>>>(reinterpret_cast<const uint4*>(sk), reinterpret_cast<const uint4*>(sv),
                                                 reinterpret_cast<uint4*>(dk), reinterpret_cast<uint4*>(dv), H,
                                                 unit_bytes / 16, r);
  return cudaGetLastError();
}

cudaError_t paged_scatter_launch(const ScatterArgs& s, const PagedRows& r, cudaStream_t st) {
  if (r.n == 0 || s.n == 0) return cudaSuccess;
  paged_scatter<<<dim3((s.n + 31) / 32, r.n * s.H), 128, 0, st>>>(s, r);
  return cudaGetLastError();
}

cudaError_t paged_append_launch(const PagedAppend& a, int esz, cudaStream_t st) {
  if (a.n == 0) return cudaSuccess;
  if (esz == 4) paged_append<float><<<a.n * a.H, 128, 0, st>>>(a);
  else paged_append<uint16_t><<<a.n * a.H, 128, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace gear
