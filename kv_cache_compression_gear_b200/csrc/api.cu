// api.cu -- the C ABI of libgear (declared in include/gear.h).
//
// Host-side validation, cache layout, workspace sizing and launch sequencing.
// Every entry point validates on the host first and enqueues nothing on error.
#include <math.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "decode.cuh"
#include "encode.cuh"

namespace gear {
__device__ int32_t g_device_status = 0;

// SM count of the current device, cached per device (host threads may fill a
// slot concurrently with the same value).
static int current_sm_count() {
  static std::atomic<int> cached[kMaxDevices];
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  const bool slot = dev >= 0 && dev < kMaxDevices;
  if (slot && (n = cached[dev].load(std::memory_order_relaxed)) > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  if (slot) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
static int esize(int dt) { return dt == GEAR_F32 ? 4 : 2; }
static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Layout {
  size_t codes, meta, oidx, oval, lfac, rfac, buf, total;
};

// token capacity per unit, rounded up so that every 32-token tile of every
// per-token array starts on a 16-byte boundary
static int round_nmax(int n_max) { return (n_max + 31) & ~31; }

static Layout cache_layout(const gear_params* p, int B, int H, int d, int n_max, int nblk_max, int dt) {
  Layout L;
  n_max = round_nmax(n_max);
  const size_t U = (size_t)B * H;
  const int k = gear_num_outliers(p->outlier_frac, d);
  const int G = d / p->group_size;
  const int W = d * p->bits / 32;
  const int rmax = p->rank > p->buffer_rank ? p->rank : p->buffer_rank;
  const int rm = rmax > 0 ? rmax : 1;
  size_t off = 0;
  L.codes = off; off = align256(off + U * n_max * W * 4);
  if (p->channel_groups)   // [U][slots][d][2] fp32, one slot per token group
    L.meta = off, off = align256(off + U * (size_t)channel_group_slots(n_max, p->group_size) * d * 8);
  else
    L.meta = off, off = align256(off + U * n_max * G * (size_t)meta_row_bytes(1, p->meta_f16));
  L.oidx = off;  off = align256(off + U * n_max * (size_t)(k > 0 ? k : 1));
  L.oval = off;  off = align256(off + U * n_max * (size_t)(k > 0 ? k : 1) * esize(dt));
  L.lfac = off;  off = align256(off + U * n_max * rm * (dt == GEAR_F32 ? 4 : 2));
  L.rfac = off;  off = align256(off + U * nblk_max * (size_t)rpad_of(rm) * d * 4);
  L.buf = off;   off = align256(off + U * (size_t)p->buffer_len * d * esize(dt));
  L.total = off;
  return L;
}

static int e_of_len(int len) {
  // floor(log2(len) / 2)
  int lg = 0;
  while ((2 << lg) <= len) ++lg;
  return lg / 2;
}

static gear_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GEAR_OK : GEAR_ERR_CUDA; }

static bool cache_ok(const gear_cache* c) {
  return c && c->codes && c->meta && c->rfac && c->buf && c->d == 128 && c->B > 0 && c->H > 0;
}

// True when caches a and b can share one batched encode: same geometry,
// dtype, codec parameters and counters.
static bool same_shape(const gear_cache* a, const gear_cache* b) {
  return a->B == b->B && a->H == b->H && a->d == b->d && a->dtype == b->dtype && a->n_max == b->n_max &&
         a->nblk_max == b->nblk_max && a->n_comp == b->n_comp && a->n_buf == b->n_buf && a->n_blk == b->n_blk &&
         memcmp(&a->p, &b->p, sizeof(gear_params)) == 0;
}

// True when k and v can serve as the K and V caches of one layer: identical
// parameters, except that K may use per-channel key groups (the KIVI-combined
// quantizer) while V keeps per-token groups.
static bool kv_params_match(const gear_cache* k, const gear_cache* v) {
  gear_params pk = k->p;
  pk.channel_groups = v->p.channel_groups;
  return v->p.channel_groups == 0 && memcmp(&pk, &v->p, sizeof(gear_params)) == 0;
}

// Encodes n tokens per unit of kvs[i] into cs[i] (i < nt <= kMaxBatch, all of
// one shape) as block `blk` at token offset t_off, in one launch per kernel.
static gear_status encode_block(gear_cache* const* cs, const void* const* kvs, int nt, int n, int t_off, int blk,
                                int rank, void* ws, size_t ws_bytes, cudaStream_t st) {
  const gear_cache* c = cs[0];
  EncodeArgs a;
  memset(&a, 0, sizeof(a));
  a.nt = nt;
  a.Uper = c->B * c->H;
  a.U = nt * a.Uper;
  a.n = n;
  a.dtype = c->dtype;
  a.bits = c->p.bits;
  a.g = c->p.group_size;
  a.k = c->k;
  a.r = rank;
  a.T = c->p.power_iters;
  a.seed = c->p.seed;
  a.t_off = t_off;
  a.blk = blk;
  a.e_blk = e_of_len(n);
  a.one_bits = 0x3F800000u;
  a.n_max = c->n_max;
  a.nblk_max = c->nblk_max;
  a.W = c->W;
  a.G = c->G;
  a.r_max = c->r_max;
  a.meta_f16 = c->p.meta_f16;
  a.ch = c->p.channel_groups;
  if (a.ch) {
    a.ch_slots = channel_group_slots(c->n_max, a.g);
    // block 0 (possibly ending in a shorter group), then whole groups per flushed block
    a.slot0 = blk == 0 ? 0 : (c->blk0_len + a.g - 1) / a.g + (t_off - c->blk0_len) / a.g;
  }
  for (int i = 0; i < nt; ++i)
    a.ten[i] = EncodeTensor{kvs[i], cs[i]->codes, cs[i]->meta, cs[i]->oidx, cs[i]->oval, cs[i]->lfac, cs[i]->rfac};
  a.tpu = (n + 127) / 128;
  a.total_tiles = (int64_t)a.U * a.tpu;
  const int sms = current_sm_count();
  a.grid_e1 = encode_grid(a, sms);
  a.maxc = encode_maxc(a.total_tiles, a.grid_e1, a.tpu);
  const size_t gbytes = align256((size_t)a.U * a.maxc * 128 * 128 * 4);
  const size_t zbytes = align256((size_t)a.U * kZSlab);
  if (!ws || ws_bytes < gbytes + zbytes || !aligned(ws, 256)) return GEAR_ERR_WORKSPACE;
  a.gram = reinterpret_cast<float*>(ws);
  a.zbuf = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + gbytes);
  return cuda_status(encode_launch(a, sms, st));
}

// workspace of one batched encode of nt tensors shaped like c, n tokens per unit
static size_t encode_ws_bytes(const gear_cache* c, int nt, int n) {
  if (!c || n <= 0 || nt <= 0) return 0;
  EncodeArgs a;
  memset(&a, 0, sizeof(a));
  a.U = nt * c->B * c->H;
  a.tpu = (n + 127) / 128;
  a.total_tiles = (int64_t)a.U * a.tpu;
  const int grid = encode_grid(a, current_sm_count());
  const int maxc = encode_maxc(a.total_tiles, grid, a.tpu);
  return align256((size_t)a.U * maxc * 128 * 128 * 4) + align256((size_t)a.U * kZSlab);
}

// ------------------------------------------------------------------ append
// One warp waits on an mbarrier that nothing arrives on; the bounded wait gives
// up after limit_ns and records GEAR_ERR_TIMEOUT (the failure-detection path
// every kernel's waits take).
__global__ void selftest_wait(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  __syncwarp();
  mbar_wait_for(&bar, 0, limit_ns);
}

template <typename T>
__global__ void append_rows(T* __restrict__ kbuf, T* __restrict__ vbuf, const T* __restrict__ kn,
                            const T* __restrict__ vn, int U, int n_b, int slot) {
  const int u = blockIdx.x, c = threadIdx.x;
  if (u >= U) return;
  kbuf[((size_t)u * n_b + slot) * 128 + c] = kn[(size_t)u * 128 + c];
  vbuf[((size_t)u * n_b + slot) * 128 + c] = vn[(size_t)u * 128 + c];
}

}  // namespace gear

using namespace gear;

extern "C" {

int32_t gear_num_outliers(float outlier_frac, int32_t d) {
  double v = (double)outlier_frac * (double)d - 1e-9;
  if (!(v > 0.0)) return 0;
  int32_t k = (int32_t)ceil(v);
  return k > d ? d : k;
}

gear_status gear_validate_params(const gear_params* p, int32_t d) {
  if (!p) return GEAR_ERR_INVALID_ARG;
  if (p->bits != 2 && p->bits != 4 && p->bits != 8) return GEAR_ERR_INVALID_ARG;
  if (p->group_size <= 0 || d <= 0 || d % p->group_size != 0 || (p->group_size * p->bits) % 32 != 0)
    return GEAR_ERR_INVALID_ARG;
  if (!(p->outlier_frac >= 0.0f && p->outlier_frac <= 0.5f)) return GEAR_ERR_INVALID_ARG;
  if (p->rank < 0 || p->rank > 16 || p->rank > d) return GEAR_ERR_INVALID_ARG;
  if (p->buffer_len < 1) return GEAR_ERR_INVALID_ARG;
  if (p->buffer_rank < 0 || p->buffer_rank > 16 || p->buffer_rank > d || p->buffer_rank > p->buffer_len)
    return GEAR_ERR_INVALID_ARG;
  if ((p->rank > 0 || p->buffer_rank > 0) && p->power_iters < 1) return GEAR_ERR_INVALID_ARG;
  if (p->power_iters < 0) return GEAR_ERR_INVALID_ARG;
  if (p->meta_f16 != 0 && p->meta_f16 != 1) return GEAR_ERR_INVALID_ARG;
  if (p->channel_groups != 0 && p->channel_groups != 1) return GEAR_ERR_INVALID_ARG;
  if (p->channel_groups) {   // whole token groups in every flushed buffer; the buffer at least one group
    if (p->buffer_len < p->group_size || p->buffer_len % p->group_size != 0) return GEAR_ERR_INVALID_ARG;
    if (p->meta_f16) return GEAR_ERR_UNSUPPORTED;
  }
  if (d != 128) return GEAR_ERR_UNSUPPORTED;
  if (p->group_size < 32) return GEAR_ERR_UNSUPPORTED;
  if (gear_num_outliers(p->outlier_frac, d) > 16) return GEAR_ERR_UNSUPPORTED;
  return GEAR_OK;
}

size_t gear_cache_bytes(const gear_params* p, int32_t B, int32_t H, int32_t d, int32_t n_max, int32_t nblk_max,
                        gear_dtype dtype) {
  if (gear_validate_params(p, d) != GEAR_OK) return 0;
  if (B <= 0 || H <= 0 || n_max <= 0 || nblk_max <= 0 || dtype < GEAR_F16 || dtype > GEAR_F32) return 0;
  if (p->meta_f16 && dtype != GEAR_F16) return 0;
  if (p->channel_groups && dtype == GEAR_F32) return 0;
  return cache_layout(p, B, H, d, n_max, nblk_max, dtype).total;
}

gear_status gear_cache_init(gear_cache* c, const gear_params* p, int32_t B, int32_t H, int32_t d, int32_t n_max,
                            int32_t nblk_max, gear_dtype dtype, void* dev, size_t bytes) {
  if (!c || !p || !dev) return GEAR_ERR_INVALID_ARG;
  gear_status s = gear_validate_params(p, d);
  if (s != GEAR_OK) return s;
  if (B <= 0 || H <= 0 || n_max <= 0 || nblk_max <= 0 || dtype < GEAR_F16 || dtype > GEAR_F32)
    return GEAR_ERR_INVALID_ARG;
  if (!aligned(dev, 256)) return GEAR_ERR_INVALID_ARG;
  if (p->meta_f16 && dtype != GEAR_F16) return GEAR_ERR_UNSUPPORTED;   // binary16 metadata of fp16 input only
  if (p->channel_groups && dtype == GEAR_F32) return GEAR_ERR_UNSUPPORTED;   // per-channel keys of 16-bit caches
  if ((size_t)B * H * round_nmax(n_max) >= ((size_t)1 << 31)) return GEAR_ERR_UNSUPPORTED;
  Layout L = cache_layout(p, B, H, d, n_max, nblk_max, dtype);
  if (bytes < L.total) return GEAR_ERR_CAPACITY;
  memset(c, 0, sizeof(*c));
  c->B = B; c->H = H; c->d = d; c->n_max = round_nmax(n_max); c->nblk_max = nblk_max; c->dtype = dtype;
  c->p = *p;
  c->k = gear_num_outliers(p->outlier_frac, d);
  c->G = d / p->group_size;
  c->W = d * p->bits / 32;
  int rmax = p->rank > p->buffer_rank ? p->rank : p->buffer_rank;
  c->r_max = rmax > 0 ? rmax : 1;
  uint8_t* base = reinterpret_cast<uint8_t*>(dev);
  c->codes = reinterpret_cast<uint32_t*>(base + L.codes);
  c->meta = reinterpret_cast<float*>(base + L.meta);
  c->oidx = base + L.oidx;
  c->oval = base + L.oval;
  c->lfac = base + L.lfac;
  c->rfac = reinterpret_cast<float*>(base + L.rfac);
  c->buf = base + L.buf;
  return GEAR_OK;
}

gear_status gear_cache_reset(gear_cache* c) {
  if (!c) return GEAR_ERR_INVALID_ARG;
  c->n_comp = c->n_buf = c->n_blk = c->blk0_len = c->blk0_rank = 0;
  return GEAR_OK;
}

size_t gear_encode_workspace_bytes(const gear_cache* c, int32_t n) { return encode_ws_bytes(c, 1, n); }

gear_status gear_encode(gear_cache* c, const void* kv, int32_t n, void* workspace, size_t ws_bytes, void* stream) {
  if (!cache_ok(c) || !kv) return GEAR_ERR_INVALID_ARG;
  if (!aligned(kv, 16)) return GEAR_ERR_INVALID_ARG;
  if (n < 1) return GEAR_ERR_INVALID_ARG;
  if (c->n_comp != 0 || c->n_buf != 0 || c->n_blk != 0) return GEAR_ERR_INVALID_ARG;
  if (c->p.rank > n) return GEAR_ERR_INVALID_ARG;
  if (n > c->n_max || c->nblk_max < 1) return GEAR_ERR_CAPACITY;
  if ((int64_t)c->B * c->H * n >= ((int64_t)1 << 31)) return GEAR_ERR_UNSUPPORTED;
  gear_status s = encode_block(&c, &kv, 1, n, 0, 0, c->p.rank, workspace, ws_bytes, (cudaStream_t)stream);
  if (s != GEAR_OK) return s;
  c->n_comp = n;
  c->n_blk = 1;
  c->blk0_len = n;
  c->blk0_rank = c->p.rank;
  return GEAR_OK;
}

size_t gear_encode_batch_workspace_bytes(int32_t count, const gear_cache* const* caches, int32_t n) {
  if (count < 1 || !caches || !caches[0]) return 0;
  return encode_ws_bytes(caches[0], count < kMaxBatch ? count : kMaxBatch, n);
}

gear_status gear_encode_batch(int32_t count, gear_cache* const* caches, const void* const* kv, int32_t n,
                              void* workspace, size_t ws_bytes, void* stream) {
  if (count < 1 || !caches || !kv || n < 1) return GEAR_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    gear_cache* c = caches[i];
    if (!cache_ok(c) || !kv[i] || !aligned(kv[i], 16)) return GEAR_ERR_INVALID_ARG;
    if (!same_shape(caches[0], c)) return GEAR_ERR_INVALID_ARG;
    for (int j = 0; j < i; ++j)
      if (caches[j] == c || caches[j]->codes == c->codes) return GEAR_ERR_INVALID_ARG;
  }
  gear_cache* c = caches[0];
  if (c->n_comp != 0 || c->n_buf != 0 || c->n_blk != 0) return GEAR_ERR_INVALID_ARG;
  if (c->p.rank > n) return GEAR_ERR_INVALID_ARG;
  if (n > c->n_max || c->nblk_max < 1) return GEAR_ERR_CAPACITY;
  if ((int64_t)c->B * c->H * n >= ((int64_t)1 << 31)) return GEAR_ERR_UNSUPPORTED;
  for (int i0 = 0; i0 < count; i0 += kMaxBatch) {
    const int nt = count - i0 < kMaxBatch ? count - i0 : kMaxBatch;
    gear_status s = encode_block(caches + i0, kv + i0, nt, n, 0, 0, c->p.rank, workspace, ws_bytes,
                                 (cudaStream_t)stream);
    if (s != GEAR_OK) return s;
  }
  for (int i = 0; i < count; ++i) {
    gear_cache* ci = caches[i];
    ci->n_comp = n;
    ci->n_blk = 1;
    ci->blk0_len = n;
    ci->blk0_rank = ci->p.rank;
  }
  return GEAR_OK;
}

static gear_status decode_args(const gear_cache* k, const gear_cache* v, int32_t Hq, DecodeArgs& a) {
  if (!cache_ok(k) || !cache_ok(v)) return GEAR_ERR_INVALID_ARG;
  if (k->B != v->B || k->H != v->H || k->dtype != v->dtype || k->n_comp != v->n_comp || k->n_buf != v->n_buf ||
      k->n_blk != v->n_blk || k->blk0_len != v->blk0_len || k->n_max != v->n_max || k->nblk_max != v->nblk_max ||
      !kv_params_match(k, v))
    return GEAR_ERR_INVALID_ARG;
  if (Hq <= 0 || Hq % k->H != 0 || Hq / k->H > 8) return GEAR_ERR_INVALID_ARG;
  if (k->n_comp + k->n_buf == 0) return GEAR_ERR_INVALID_ARG;
  memset(&a, 0, sizeof(a));
  a.K = CacheView{k->codes, k->meta, k->oidx, k->oval, k->lfac, k->rfac, k->buf};
  a.V = CacheView{v->codes, v->meta, v->oidx, v->oval, v->lfac, v->rfac, v->buf};
  a.dtype = k->dtype;
  a.B = k->B; a.H = k->H; a.Hq = Hq; a.hq = Hq / k->H;
  a.bits = k->p.bits; a.g = k->p.group_size; a.G = k->G; a.W = k->W; a.k = k->k; a.r_max = k->r_max;
  a.meta_f16 = k->p.meta_f16;
  a.kc = k->p.channel_groups;
  a.ch_slots = a.kc ? channel_group_slots(k->n_max, k->p.group_size) : 0;
  if (a.kc && a.hq > 4) return GEAR_ERR_UNSUPPORTED;   // per-channel key groups: up to 4 query heads per kv head
  a.n_max = k->n_max; a.nblk_max = k->nblk_max; a.n_b = k->p.buffer_len;
  a.n_comp = k->n_comp; a.n_buf = k->n_buf;
  a.blk0_len = k->blk0_len; a.blk0_rank = k->blk0_rank; a.buffer_rank = k->p.buffer_rank;
  decode_plan(a, current_sm_count());
  return GEAR_OK;
}

size_t gear_decode_workspace_bytes(const gear_cache* k, const gear_cache* v, int32_t Hq) {
  DecodeArgs a;
  if (decode_args(k, v, Hq, a) != GEAR_OK) return 0;
  return decode_workspace_bytes(a.B, a.Hq, a.nsplit);
}

static gear_status decode_attn(const gear_cache* k, const gear_cache* v, const void* q, int32_t Hq,
                               float softmax_scale, void* out, gear_dtype out_dtype, const int32_t* prefill_len,
                               void* workspace, size_t ws_bytes, void* stream) {
  DecodeArgs a;
  gear_status s = decode_args(k, v, Hq, a);
  if (s != GEAR_OK) return s;
  a.plen = prefill_len;
  if (!q || !out) return GEAR_ERR_INVALID_ARG;
  if (out_dtype != k->dtype && out_dtype != GEAR_F32) return GEAR_ERR_INVALID_ARG;
  if (!isfinite(softmax_scale)) return GEAR_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < decode_workspace_bytes(a.B, a.Hq, a.nsplit) || !aligned(workspace, 16))
    return GEAR_ERR_WORKSPACE;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.one_bits = 0x3F800000u;
  a.q = q;
  a.out = out;
  a.out_dtype = out_dtype;
  a.part = reinterpret_cast<float*>(workspace);
  return cuda_status(decode_launch(a, (cudaStream_t)stream));
}

gear_status gear_decode_attn(const gear_cache* k, const gear_cache* v, const void* q, int32_t Hq, float softmax_scale,
                             void* out, gear_dtype out_dtype, void* workspace, size_t ws_bytes, void* stream) {
  return decode_attn(k, v, q, Hq, softmax_scale, out, out_dtype, nullptr, workspace, ws_bytes, stream);
}

gear_status gear_decode_attn_ragged(const gear_cache* k, const gear_cache* v, const void* q, int32_t Hq,
                                    float softmax_scale, void* out, gear_dtype out_dtype, const int32_t* prefill_len,
                                    void* workspace, size_t ws_bytes, void* stream) {
  if (!prefill_len || !aligned(prefill_len, 4)) return GEAR_ERR_INVALID_ARG;
  return decode_attn(k, v, q, Hq, softmax_scale, out, out_dtype, prefill_len, workspace, ws_bytes, stream);
}

size_t gear_append_workspace_bytes(const gear_cache* k) {
  if (!cache_ok(k)) return 0;
  return encode_ws_bytes(k, 2, k->p.buffer_len);
}

gear_status gear_append_buffer(gear_cache* k, gear_cache* v, const void* k_new, const void* v_new, void* workspace,
                               size_t ws_bytes, void* stream) {
  if (!cache_ok(k) || !cache_ok(v) || !k_new || !v_new) return GEAR_ERR_INVALID_ARG;
  if (k->B != v->B || k->H != v->H || k->dtype != v->dtype || k->n_comp != v->n_comp || k->n_buf != v->n_buf ||
      k->n_blk != v->n_blk || !kv_params_match(k, v))
    return GEAR_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const int n_b = k->p.buffer_len;
  const bool flush = k->n_buf == n_b;
  if (flush) {
    if (k->n_comp + n_b > k->n_max || k->n_blk + 1 > k->nblk_max) return GEAR_ERR_CAPACITY;
    gear_cache* cs[2] = {k, v};
    const void* bufs[2] = {k->buf, v->buf};
    if (same_shape(k, v)) {   // both tensors in one pass
      if (ws_bytes < encode_ws_bytes(k, 2, n_b)) return GEAR_ERR_WORKSPACE;
      gear_status s = encode_block(cs, bufs, 2, n_b, k->n_comp, k->n_blk, k->p.buffer_rank, workspace, ws_bytes, st);
      if (s != GEAR_OK) return s;
    } else {
      if (ws_bytes < encode_ws_bytes(k, 1, n_b)) return GEAR_ERR_WORKSPACE;
      for (int i = 0; i < 2; ++i) {
        gear_status s = encode_block(&cs[i], &bufs[i], 1, n_b, cs[i]->n_comp, cs[i]->n_blk, cs[i]->p.buffer_rank,
                                     workspace, ws_bytes, st);
        if (s != GEAR_OK) return s;
      }
    }
    for (gear_cache* c : cs) {
      if (c->n_blk == 0) { c->blk0_len = n_b; c->blk0_rank = c->p.buffer_rank; }
      c->n_comp += n_b;
      c->n_blk += 1;
      c->n_buf = 0;
    }
  }
  const int U = k->B * k->H;
  if (k->dtype == GEAR_F32)
    append_rows<float><<<U, 128, 0, st>>>((float*)k->buf, (float*)v->buf, (const float*)k_new, (const float*)v_new, U,
                                          n_b, k->n_buf);
  else
    append_rows<uint16_t><<<U, 128, 0, st>>>((uint16_t*)k->buf, (uint16_t*)v->buf, (const uint16_t*)k_new,
                                             (const uint16_t*)v_new, U, n_b, k->n_buf);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return GEAR_ERR_CUDA;
  k->n_buf += 1;
  v->n_buf += 1;
  return GEAR_OK;
}

gear_status gear_decode_dense(const gear_cache* c, float* out_f32, void* stream) {
  if (!cache_ok(c) || !out_f32) return GEAR_ERR_INVALID_ARG;
  DenseArgs a;
  memset(&a, 0, sizeof(a));
  a.C = CacheView{c->codes, c->meta, c->oidx, c->oval, c->lfac, c->rfac, c->buf};
  a.dtype = c->dtype;
  a.U = c->B * c->H;
  a.bits = c->p.bits; a.g = c->p.group_size; a.G = c->G; a.W = c->W; a.k = c->k; a.r_max = c->r_max;
  a.meta_f16 = c->p.meta_f16;
  a.ch = c->p.channel_groups;
  a.ch_slots = a.ch ? channel_group_slots(c->n_max, c->p.group_size) : 0;
  a.n_max = c->n_max; a.nblk_max = c->nblk_max; a.n_b = c->p.buffer_len;
  a.n_comp = c->n_comp; a.n_buf = c->n_buf;
  a.blk0_len = c->blk0_len; a.blk0_rank = c->blk0_rank; a.buffer_rank = c->p.buffer_rank;
  a.out = out_f32;
  return cuda_status(dense_launch(a, (cudaStream_t)stream));
}

gear_status gear_get_device_status(int32_t* status) {
  if (!status) return GEAR_ERR_INVALID_ARG;
  int32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return GEAR_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return GEAR_ERR_CUDA;
  *status = v;
  return GEAR_OK;
}

gear_status gear_selftest_wait_timeout(uint32_t limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return GEAR_ERR_INVALID_ARG;
  selftest_wait<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_us * 1000ull);
  return cuda_status(cudaGetLastError());
}

const char* gear_status_string(gear_status s) {
  switch (s) {
    case GEAR_OK: return "ok";
    case GEAR_ERR_INVALID_ARG: return "invalid argument";
    case GEAR_ERR_UNSUPPORTED: return "unsupported configuration";
    case GEAR_ERR_CAPACITY: return "cache capacity exceeded";
    case GEAR_ERR_CUDA: return "CUDA runtime error";
    case GEAR_ERR_TIMEOUT: return "device-side wait timed out";
    case GEAR_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

const char* gear_version(void) { return "0.1.0"; }

}  // extern "C"

// ------------------------------------------------------------------ no-alloc decode
// Decode attention for callers that cannot call cudaMalloc. The split-K
// partial results live in a fixed array inside this library instead of a
// caller-provided workspace. The array is a file-scope __device__ variable, so
// every GPU that loads the library holds it (4 MiB) until the process exits.
// Host code cannot pass the array's name to a kernel (in host code it is a
// host-side stand-in), so its device address is looked up once per device
// with cudaGetSymbolAddress and cached.
namespace gear {
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

static std::mutex g_noalloc_mu;
static float* g_noalloc_ptr[256];

// Device address of the scratch array on the current device (nullptr on error).
static float* noalloc_scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
    g_noalloc_ptr[dev] = reinterpret_cast<float*>(p);
  }
  return g_noalloc_ptr[dev];
}
}  // namespace gear

extern "C" gear_status gear_decode_attn_noalloc(const gear_cache* k, const gear_cache* v, const void* q, int32_t Hq,
                                                float softmax_scale, void* out, gear_dtype out_dtype, void* stream) {
  DecodeArgs a;
  gear_status s = decode_args(k, v, Hq, a);
  if (s != GEAR_OK) return s;
  if (!q || !out) return GEAR_ERR_INVALID_ARG;
  if (out_dtype != k->dtype && out_dtype != GEAR_F32) return GEAR_ERR_INVALID_ARG;
  if (!isfinite(softmax_scale)) return GEAR_ERR_INVALID_ARG;
  if (decode_workspace_bytes(a.B, a.Hq, a.nsplit) > kNoAllocScratchBytes) return GEAR_ERR_WORKSPACE;
  float* scratch = noalloc_scratch_for_current_device();
  if (!scratch) return GEAR_ERR_CUDA;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.one_bits = 0x3F800000u;
  a.q = q;
  a.out = out;
  a.out_dtype = out_dtype;
  a.part = scratch;  // every split writes all of its partial row: nothing needs clearing
  return cuda_status(decode_launch(a, (cudaStream_t)stream));
}
