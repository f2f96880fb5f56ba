// api.cu -- the C ABI of libgear (declared in include/gear.h).
//
// Host-side validation, cache layout, workspace sizing and launch sequencing.
// Every entry point validates on the host first and enqueues nothing on error.
#include <math.h>
#include <string.h>

#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "decode.cuh"
#include "encode.cuh"
#include "paged.cuh"

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

// Layout of U units whose per-token arrays hold tok_rows rows in all (U * n_max
// in a contiguous cache, num_pages * H * P in a paged pool); ch_slots > 0 gives
// the per-channel key meta of U * ch_slots token groups instead.
static Layout layout_rows(const gear_params* p, size_t U, size_t tok_rows, size_t ch_slots, int d, int nblk_max,
                          int dt) {
  Layout L;
  const int k = gear_num_outliers(p->outlier_frac, d);
  const int G = d / p->group_size;
  const int W = d * p->bits / 32;
  const int rmax = p->rank > p->buffer_rank ? p->rank : p->buffer_rank;
  const int rm = rmax > 0 ? rmax : 1;
  size_t off = 0;
  L.codes = off; off = align256(off + tok_rows * W * 4);
  if (ch_slots)   // [U][slots][d][2] fp32, one slot per token group
    L.meta = off, off = align256(off + U * ch_slots * d * 8);
  else
    L.meta = off, off = align256(off + tok_rows * G * (size_t)meta_row_bytes(1, p->meta_f16));
  L.oidx = off;  off = align256(off + tok_rows * (size_t)(k > 0 ? k : 1));
  L.oval = off;  off = align256(off + tok_rows * (size_t)(k > 0 ? k : 1) * esize(dt));
  L.lfac = off;  off = align256(off + tok_rows * rm * (dt == GEAR_F32 ? 4 : 2));
  L.rfac = off;  off = align256(off + U * nblk_max * (size_t)rpad_of(rm) * d * 4);
  L.buf = off;   off = align256(off + U * (size_t)p->buffer_len * d * esize(dt));
  L.total = off;
  return L;
}

static Layout cache_layout(const gear_params* p, int B, int H, int d, int n_max, int nblk_max, int dt) {
  n_max = round_nmax(n_max);
  const size_t U = (size_t)B * H;
  const size_t slots = p->channel_groups ? (size_t)channel_group_slots(n_max, p->group_size) : 0;
  return layout_rows(p, U, U * n_max, slots, d, nblk_max, dt);
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

// ------------------------------------------------------------------ paged layout
// Host state of a paged cache, in the caller's int32 array: per-row counters,
// the mirror of the device block table and a stack of free pool pages.
struct HostView {
  int32_t* b0;     // [B] block-0 length
  int32_t* nblk;   // [B] blocks (0: empty row)
  int32_t* nbuf;   // [B] buffer fill
  int32_t* table;  // [B][ppr] pool page of each logical page, -1 if none
  int32_t* stack;  // [num_pages] free pages, top at stack[*top - 1]
  int32_t* top;    // number of free pages
};

static size_t paged_host_ints(int B, int ppr, int num_pages) {
  return 3 * (size_t)B + (size_t)B * ppr + (size_t)num_pages + 1;
}

static HostView host_view(const gear_cache* c) {
  HostView h;
  int32_t* p = c->host;
  h.b0 = p;
  h.nblk = p + c->B;
  h.nbuf = p + 2 * (size_t)c->B;
  h.table = p + 3 * (size_t)c->B;
  h.stack = h.table + (size_t)c->B * c->pages_per_row;
  h.top = h.stack + c->num_pages;
  return h;
}

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

static int row_ncomp(const gear_cache* c, const HostView& h, int b) {
  return h.nblk[b] > 0 ? h.b0[b] + (h.nblk[b] - 1) * c->p.buffer_len : 0;
}

static bool is_paged(const gear_cache* c) { return c && c->page_tokens > 0; }

static bool paged_ok(const gear_cache* c) {
  return cache_ok(c) && c->page_tokens > 0 && c->num_pages > 0 && c->pages_per_row > 0 && c->host && c->table &&
         c->rows;
}

// K and V caches built by the same calls: same geometry, parameters and host
// state, so that one table serves both. Compared: the row counters, the table
// entries in use (a row holds exactly the pages its tokens reach) and the free
// stack, O(B + num_pages) per call.
static bool paged_pair(const gear_cache* k, const gear_cache* v) {
  if (!(k->B == v->B && k->H == v->H && k->dtype == v->dtype && k->page_tokens == v->page_tokens &&
        k->num_pages == v->num_pages && k->pages_per_row == v->pages_per_row && k->nblk_max == v->nblk_max &&
        k->n_comp == v->n_comp && k->n_buf == v->n_buf && k->n_blk == v->n_blk && kv_params_match(k, v)))
    return false;
  const int B = k->B;
  if (memcmp(k->host, v->host, (size_t)3 * B * sizeof(int32_t)) != 0) return false;
  const HostView hk = host_view(k), hv = host_view(v);
  for (int b = 0; b < B; ++b) {
    const size_t used = (size_t)((row_ncomp(k, hk, b) + k->page_tokens - 1) / k->page_tokens);
    const size_t off = (size_t)b * k->pages_per_row;
    if (used && memcmp(hk.table + off, hv.table + off, used * sizeof(int32_t)) != 0) return false;
  }
  return *hk.top == *hv.top && memcmp(hk.stack, hv.stack, (size_t)*hk.top * sizeof(int32_t)) == 0;
}

// rows[0 .. nrows) are distinct rows of c
static bool rows_ok(const gear_cache* c, const int32_t* rows, int nrows) {
  if (!rows || nrows < 1 || nrows > c->B) return false;
  std::vector<char> seen((size_t)c->B, 0);
  for (int i = 0; i < nrows; ++i) {
    if (rows[i] < 0 || rows[i] >= c->B || seen[rows[i]]) return false;
    seen[rows[i]] = 1;
  }
  return true;
}

static void update_maxima(gear_cache* c) {
  HostView h = host_view(c);
  int nc = 0, nb = 0, nk = 0;
  for (int b = 0; b < c->B; ++b) {
    const int r = row_ncomp(c, h, b);
    nc = r > nc ? r : nc;
    nb = h.nbuf[b] > nb ? h.nbuf[b] : nb;
    nk = h.nblk[b] > nk ? h.nblk[b] : nk;
  }
  c->n_comp = nc;
  c->n_buf = nb;
  c->n_blk = nk;
}

struct RowState {
  int32_t row, b0, nblk, nbuf;
};

// Writes table entries (index, page) and row states to the device, in
// launches of paged_set.
static cudaError_t enqueue_set(const gear_cache* c, const std::vector<std::pair<int, int>>& tab,
                               const std::vector<RowState>& rs, cudaStream_t st) {
  size_t it = 0, ir = 0;
  while (it < tab.size() || ir < rs.size()) {
    PagedSet s;
    memset(&s, 0, sizeof(s));
    s.table = c->table;
    s.rows = c->rows;
    s.B = c->B;
    for (; it < tab.size() && s.ntab < kSetMax; ++it, ++s.ntab) {
      s.tab_idx[s.ntab] = tab[it].first;
      s.tab_val[s.ntab] = tab[it].second;
    }
    for (; ir < rs.size() && s.nrow < kSetRows; ++ir, ++s.nrow) {
      s.row[s.nrow] = rs[ir].row;
      s.b0[s.nrow] = rs[ir].b0;
      s.nblk[s.nrow] = rs[ir].nblk;
      s.nbuf[s.nrow] = rs[ir].nbuf;
    }
    cudaError_t e = paged_set_launch(s, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Moves n tokens per unit of the staging cache stg (rows i of the call are its
// batch rows i) into the pages of c: row rows[i] at token offset t0[i], block
// blk[i]. The device table must already map every page these tokens reach.
static cudaError_t scatter_rows(const gear_cache* c, const gear_cache* stg, const int32_t* rows, const int* t0,
                                const int* blk, const int* s0, int nrows, int n, cudaStream_t st) {
  ScatterArgs s;
  memset(&s, 0, sizeof(s));
  s.s_codes = reinterpret_cast<const uint8_t*>(stg->codes);
  s.s_meta = reinterpret_cast<const uint8_t*>(stg->meta);
  s.s_oidx = stg->oidx;
  s.s_oval = reinterpret_cast<const uint8_t*>(stg->oval);
  s.s_lfac = reinterpret_cast<const uint8_t*>(stg->lfac);
  s.s_rfac = stg->rfac;
  s.d_codes = reinterpret_cast<uint8_t*>(c->codes);
  s.d_meta = reinterpret_cast<uint8_t*>(c->meta);
  s.d_oidx = c->oidx;
  s.d_oval = reinterpret_cast<uint8_t*>(c->oval);
  s.d_lfac = reinterpret_cast<uint8_t*>(c->lfac);
  s.d_rfac = c->rfac;
  s.table = c->table;
  s.H = c->H;
  s.P = c->page_tokens;
  s.ppr = c->pages_per_row;
  s.num_pages = c->num_pages;
  s.nblk_max = c->nblk_max;
  s.nmax_s = stg->n_max;
  s.n = n;
  s.wb = c->W * 4;
  s.ch = c->p.channel_groups;
  s.mb = s.ch ? 0 : meta_row_bytes(c->G, c->p.meta_f16);
  s.g = c->p.group_size;
  s.ch_slots_s = s.ch ? channel_group_slots(stg->n_max, s.g) : 0;
  s.ch_slots_d = s.ch ? channel_group_slots(c->n_max, s.g) : 0;
  s.kb = c->k;
  s.ob = c->k * esize(c->dtype);
  s.lb = c->r_max * (c->dtype == GEAR_F32 ? 4 : 2);
  s.rf_floats = 128 * rpad_of(c->r_max);
  for (int i0 = 0; i0 < nrows; i0 += kRowsMax) {
    PagedRows r;
    memset(&r, 0, sizeof(r));
    r.n = nrows - i0 < kRowsMax ? nrows - i0 : kRowsMax;
    r.i0 = i0;
    for (int j = 0; j < r.n; ++j) {
      r.row[j] = rows[i0 + j];
      r.t0[j] = t0[i0 + j];
      r.blk[j] = blk[i0 + j];
      r.s0[j] = s0[i0 + j];
    }
    cudaError_t e = paged_scatter_launch(s, r, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Bytes of a contiguous staging cache of nrows rows and n tokens (one block).
static size_t staging_bytes(const gear_cache* c, int nrows, int n) {
  return align256(cache_layout(&c->p, nrows, c->H, c->d, n, 1, c->dtype).total);
}

// encode workspace of nt tensors of nrows rows shaped like c, n tokens per unit
static size_t rows_encode_ws(const gear_cache* c, int nt, int nrows, int n) {
  gear_cache t = *c;
  t.B = nrows;
  return encode_ws_bytes(&t, nt, n);
}

// workspace of a flush of nf rows (K and V): two staging caches, the gathered
// buffers and the batched encode
// (V's parameters are K's with channel_groups = 0: kv_params_match)
static size_t flush_ws_bytes(const gear_cache* k, int nf) {
  const int n_b = k->p.buffer_len;
  const size_t in = align256((size_t)nf * k->H * n_b * k->d * esize(k->dtype));
  gear_cache v = *k;
  v.p.channel_groups = 0;
  return staging_bytes(k, nf, n_b) + staging_bytes(&v, nf, n_b) + 2 * in + rows_encode_ws(k, 2, nf, n_b);
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
  if (is_paged(c)) return GEAR_ERR_UNSUPPORTED;   // rows are released one by one
  c->n_comp = c->n_buf = c->n_blk = c->blk0_len = c->blk0_rank = 0;
  return GEAR_OK;
}

size_t gear_encode_workspace_bytes(const gear_cache* c, int32_t n) { return encode_ws_bytes(c, 1, n); }

gear_status gear_encode(gear_cache* c, const void* kv, int32_t n, void* workspace, size_t ws_bytes, void* stream) {
  if (!cache_ok(c) || !kv) return GEAR_ERR_INVALID_ARG;
  if (is_paged(c)) return GEAR_ERR_UNSUPPORTED;
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
    if (is_paged(c)) return GEAR_ERR_UNSUPPORTED;
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
  if (is_paged(k) != is_paged(v)) return GEAR_ERR_INVALID_ARG;
  if (is_paged(k) && (!paged_ok(k) || !paged_ok(v) || !paged_pair(k, v))) return GEAR_ERR_INVALID_ARG;
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
  if (is_paged(k)) {   // one table serves both tensors (paged_pair: equal host state)
    a.table = k->table;
    a.rows = k->rows;
    a.page_tokens = k->page_tokens;
    a.ppr = k->pages_per_row;
    a.num_pages = k->num_pages;
    // the split runs over the tokens the rows hold, not over B * H * max length
    const HostView h = host_view(k);
    int64_t tot = 0;
    for (int b = 0; b < k->B; ++b) tot += (int64_t)k->H * row_ncomp(k, h, b);
    a.tot_tokens = tot;
  }
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
  if (is_paged(k) || is_paged(v)) return GEAR_ERR_UNSUPPORTED;
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
  if (is_paged(c)) return GEAR_ERR_UNSUPPORTED;
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

// ------------------------------------------------------------------ paged layout
size_t gear_paged_host_ints(int32_t B, int32_t pages_per_row, int32_t num_pages) {
  if (B <= 0 || pages_per_row <= 0 || num_pages <= 0) return 0;
  return paged_host_ints(B, pages_per_row, num_pages);
}

static gear_status paged_geometry(const gear_params* p, int32_t B, int32_t H, int32_t d, int32_t P, int32_t num_pages,
                                  int32_t ppr, int32_t nblk_max, gear_dtype dtype) {
  gear_status s = gear_validate_params(p, d);
  if (s != GEAR_OK) return s;
  if (B <= 0 || H <= 0 || P <= 0 || P % 32 != 0 || num_pages <= 0 || ppr <= 0 || nblk_max <= 0 ||
      dtype < GEAR_F16 || dtype > GEAR_F32)
    return GEAR_ERR_INVALID_ARG;
  if (p->meta_f16 && dtype != GEAR_F16) return GEAR_ERR_UNSUPPORTED;
  if (p->channel_groups && dtype == GEAR_F32) return GEAR_ERR_UNSUPPORTED;   // per-channel keys of 16-bit caches
  if ((int64_t)num_pages * H * P >= ((int64_t)1 << 31) || (int64_t)P * ppr >= ((int64_t)1 << 31) ||
      (int64_t)B * ppr >= ((int64_t)1 << 31))
    return GEAR_ERR_UNSUPPORTED;
  return GEAR_OK;
}

static size_t paged_total(const gear_params* p, int B, int H, int d, int P, int num_pages, int ppr, int nblk_max,
                          int dt, Layout* L, size_t* table_off, size_t* rows_off) {
  // per-channel key groups: the meta slots stay per unit, for a row's whole capacity
  const size_t slots = p->channel_groups ? (size_t)channel_group_slots(P * ppr, p->group_size) : 0;
  *L = layout_rows(p, (size_t)B * H, (size_t)num_pages * H * P, slots, d, nblk_max, dt);
  *table_off = L->total;
  *rows_off = *table_off + align256((size_t)B * ppr * 4);
  return *rows_off + align256((size_t)3 * B * 4);
}

size_t gear_paged_cache_bytes(const gear_params* p, int32_t B, int32_t H, int32_t d, int32_t page_tokens,
                              int32_t num_pages, int32_t pages_per_row, int32_t nblk_max, gear_dtype dtype) {
  if (paged_geometry(p, B, H, d, page_tokens, num_pages, pages_per_row, nblk_max, dtype) != GEAR_OK) return 0;
  Layout L;
  size_t to, ro;
  return paged_total(p, B, H, d, page_tokens, num_pages, pages_per_row, nblk_max, dtype, &L, &to, &ro);
}

gear_status gear_paged_cache_init(gear_cache* c, const gear_params* p, int32_t B, int32_t H, int32_t d,
                                  int32_t page_tokens, int32_t num_pages, int32_t pages_per_row, int32_t nblk_max,
                                  gear_dtype dtype, void* dev, size_t bytes, int32_t* host, size_t host_ints,
                                  void* stream) {
  if (!c || !p || !dev || !host) return GEAR_ERR_INVALID_ARG;
  if (!aligned(dev, 256)) return GEAR_ERR_INVALID_ARG;
  gear_status s = paged_geometry(p, B, H, d, page_tokens, num_pages, pages_per_row, nblk_max, dtype);
  if (s != GEAR_OK) return s;
  Layout L;
  size_t to, ro;
  const size_t total = paged_total(p, B, H, d, page_tokens, num_pages, pages_per_row, nblk_max, dtype, &L, &to, &ro);
  if (bytes < total || host_ints < paged_host_ints(B, pages_per_row, num_pages)) return GEAR_ERR_CAPACITY;
  memset(c, 0, sizeof(*c));
  c->B = B; c->H = H; c->d = d; c->n_max = page_tokens * pages_per_row; c->nblk_max = nblk_max; c->dtype = dtype;
  c->p = *p;
  c->k = gear_num_outliers(p->outlier_frac, d);
  c->G = d / p->group_size;
  c->W = d * p->bits / 32;
  const int rmax = p->rank > p->buffer_rank ? p->rank : p->buffer_rank;
  c->r_max = rmax > 0 ? rmax : 1;
  c->blk0_rank = p->rank;
  uint8_t* base = reinterpret_cast<uint8_t*>(dev);
  c->codes = reinterpret_cast<uint32_t*>(base + L.codes);
  c->meta = reinterpret_cast<float*>(base + L.meta);
  c->oidx = base + L.oidx;
  c->oval = base + L.oval;
  c->lfac = base + L.lfac;
  c->rfac = reinterpret_cast<float*>(base + L.rfac);
  c->buf = base + L.buf;
  c->page_tokens = page_tokens;
  c->num_pages = num_pages;
  c->pages_per_row = pages_per_row;
  c->table = reinterpret_cast<int32_t*>(base + to);
  c->rows = reinterpret_cast<int32_t*>(base + ro);
  c->host = host;
  HostView h = host_view(c);
  for (int b = 0; b < 3 * B; ++b) host[b] = 0;
  for (size_t i = 0; i < (size_t)B * pages_per_row; ++i) h.table[i] = -1;
  for (int i = 0; i < num_pages; ++i) h.stack[i] = num_pages - 1 - i;   // page 0 is handed out first
  *h.top = num_pages;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemsetAsync(c->rows, 0, (size_t)3 * B * 4, st) != cudaSuccess ||
      cudaMemsetAsync(c->table, 0xFF, (size_t)B * pages_per_row * 4, st) != cudaSuccess)
    return GEAR_ERR_CUDA;
  return GEAR_OK;
}

size_t gear_encode_rows_workspace_bytes(const gear_cache* c, int32_t nrows, int32_t n) {
  if (!paged_ok(c) || nrows < 1 || nrows > c->B || n < 1) return 0;
  return staging_bytes(c, nrows, n) + rows_encode_ws(c, 1, nrows, n);
}

gear_status gear_encode_rows(gear_cache* c, const int32_t* rows, int32_t nrows, const void* kv, int32_t n,
                             void* workspace, size_t ws_bytes, void* stream) {
  if (!paged_ok(c) || !kv || !aligned(kv, 16) || n < 1) return GEAR_ERR_INVALID_ARG;
  if (!rows_ok(c, rows, nrows)) return GEAR_ERR_INVALID_ARG;
  HostView h = host_view(c);
  for (int i = 0; i < nrows; ++i)
    if (h.nblk[rows[i]] != 0 || h.nbuf[rows[i]] != 0) return GEAR_ERR_INVALID_ARG;
  if (c->p.rank > n) return GEAR_ERR_INVALID_ARG;
  const int P = c->page_tokens, per = ceil_div(n, P);
  if (n > c->n_max) return GEAR_ERR_CAPACITY;
  if ((int64_t)per * nrows > *h.top) return GEAR_ERR_CAPACITY;
  if ((int64_t)nrows * c->H * n >= ((int64_t)1 << 31)) return GEAR_ERR_UNSUPPORTED;
  const size_t sb = staging_bytes(c, nrows, n);
  if (!workspace || !aligned(workspace, 256) || ws_bytes < sb + rows_encode_ws(c, 1, nrows, n))
    return GEAR_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  // the codec on a contiguous copy of the rows
  gear_cache stg;
  gear_status s = gear_cache_init(&stg, &c->p, nrows, c->H, c->d, n, 1, (gear_dtype)c->dtype, workspace, sb);
  if (s != GEAR_OK) return s;
  gear_cache* sp = &stg;
  s = encode_block(&sp, &kv, 1, n, 0, 0, c->p.rank, reinterpret_cast<uint8_t*>(workspace) + sb, ws_bytes - sb, st);
  if (s != GEAR_OK) return s;
  // pages for tokens [0, n) of every row, then the move into them
  std::vector<std::pair<int, int>> tab;
  std::vector<RowState> rs;
  std::vector<int> t0((size_t)nrows, 0), blk((size_t)nrows, 0), s0((size_t)nrows, 0);
  for (int i = 0; i < nrows; ++i) {
    const int b = rows[i];
    for (int lp = 0; lp < per; ++lp) {
      const int pg = h.stack[--*h.top];
      h.table[(size_t)b * c->pages_per_row + lp] = pg;
      tab.emplace_back(b * c->pages_per_row + lp, pg);
    }
    h.b0[b] = n;
    h.nblk[b] = 1;
    h.nbuf[b] = 0;
    rs.push_back(RowState{b, n, 1, 0});
  }
  update_maxima(c);
  cudaError_t e = enqueue_set(c, tab, rs, st);
  if (e == cudaSuccess) e = scatter_rows(c, &stg, rows, t0.data(), blk.data(), s0.data(), nrows, n, st);
  return cuda_status(e);
}

size_t gear_append_rows_workspace_bytes(const gear_cache* k) {
  if (!paged_ok(k)) return 0;
  size_t m = 0;
  for (int nf = 1; nf <= k->B; ++nf) {   // the encode's partial-Gram slots depend on the row count
    const size_t b = flush_ws_bytes(k, nf);
    m = b > m ? b : m;
  }
  return m;
}

gear_status gear_append_rows(gear_cache* k, gear_cache* v, const int32_t* rows, int32_t nrows, const void* k_new,
                             const void* v_new, void* workspace, size_t ws_bytes, void* stream) {
  if (!paged_ok(k) || !paged_ok(v) || k == v || !k_new || !v_new) return GEAR_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return GEAR_ERR_INVALID_ARG;
  if (!paged_pair(k, v) || !rows_ok(k, rows, nrows)) return GEAR_ERR_INVALID_ARG;
  HostView hk = host_view(k), hv = host_view(v);
  const int n_b = k->p.buffer_len, P = k->page_tokens;
  std::vector<int32_t> fr;   // rows whose buffer is flushed first
  std::vector<int> ft0, fblk, fs0;   // token offset, block and (per-channel keys) first slot of each
  int need = 0;
  for (int i = 0; i < nrows; ++i) {
    const int b = rows[i];
    if (hk.nblk[b] == 0) return GEAR_ERR_INVALID_ARG;   // encode the row's prompt first
    if (hk.nbuf[b] == n_b) {
      const int nc = row_ncomp(k, hk, b);
      if (nc + n_b > k->n_max || hk.nblk[b] + 1 > k->nblk_max) return GEAR_ERR_CAPACITY;
      need += ceil_div(nc + n_b, P) - ceil_div(nc, P);
      fr.push_back(b);
      ft0.push_back(nc);
      fblk.push_back(hk.nblk[b]);
      // block j >= 1 starts at group slot ceil(b0 / g) + (j - 1) * n_b / g
      const int g = k->p.group_size;
      fs0.push_back(ceil_div(hk.b0[b], g) + (hk.nblk[b] - 1) * (n_b / g));
    }
  }
  if (need > *hk.top) return GEAR_ERR_CAPACITY;
  const int nf = (int)fr.size();
  if (nf > 0 && (!workspace || !aligned(workspace, 256) || ws_bytes < flush_ws_bytes(k, nf)))
    return GEAR_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  if (nf > 0) {
    // gather the full buffers, encode them as one block per row (both tensors
    // in one pass when their parameters agree), then move the blocks into fresh pages
    uint8_t* w = reinterpret_cast<uint8_t*>(workspace);
    const size_t sbk = staging_bytes(k, nf, n_b), sbv = staging_bytes(v, nf, n_b);
    const size_t ub = (size_t)k->H * n_b * k->d * esize(k->dtype);   // buffer bytes per row
    const size_t in = align256((size_t)nf * ub);
    gear_cache stk, stv;
    gear_status s = gear_cache_init(&stk, &k->p, nf, k->H, k->d, n_b, 1, (gear_dtype)k->dtype, w, sbk);
    if (s == GEAR_OK) s = gear_cache_init(&stv, &v->p, nf, v->H, v->d, n_b, 1, (gear_dtype)v->dtype, w + sbk, sbv);
    if (s != GEAR_OK) return s;
    uint8_t* ink = w + sbk + sbv;
    uint8_t* inv = ink + in;
    for (int i0 = 0; i0 < nf && e == cudaSuccess; i0 += kRowsMax) {
      PagedRows r;
      memset(&r, 0, sizeof(r));
      r.n = nf - i0 < kRowsMax ? nf - i0 : kRowsMax;
      r.i0 = i0;
      for (int j = 0; j < r.n; ++j) r.row[j] = fr[i0 + j];
      e = paged_gather_launch(k->buf, v->buf, ink, inv, k->H, (int)(ub / k->H), r, st);
    }
    if (e != cudaSuccess) return GEAR_ERR_CUDA;
    gear_cache* cs[2] = {&stk, &stv};
    const void* ins[2] = {ink, inv};
    const size_t used = sbk + sbv + 2 * in;
    if (memcmp(&k->p, &v->p, sizeof(gear_params)) == 0) {
      s = encode_block(cs, ins, 2, n_b, 0, 0, k->p.buffer_rank, inv + in, ws_bytes - used, st);
    } else {   // per-channel key groups on K only: one encode per tensor
      s = encode_block(&cs[0], &ins[0], 1, n_b, 0, 0, k->p.buffer_rank, inv + in, ws_bytes - used, st);
      if (s == GEAR_OK) s = encode_block(&cs[1], &ins[1], 1, n_b, 0, 0, v->p.buffer_rank, inv + in, ws_bytes - used, st);
    }
    if (s != GEAR_OK) return s;
    std::vector<std::pair<int, int>> tab;
    for (int i = 0; i < nf; ++i) {
      const int b = fr[i];
      for (int lp = ceil_div(ft0[i], P); lp < ceil_div(ft0[i] + n_b, P); ++lp) {
        const int pg = hk.stack[--*hk.top];
        --*hv.top;
        hk.table[(size_t)b * k->pages_per_row + lp] = pg;
        hv.table[(size_t)b * v->pages_per_row + lp] = pg;
        tab.emplace_back(b * k->pages_per_row + lp, pg);
      }
      hk.nblk[b] += 1;
      hv.nblk[b] += 1;
      hk.nbuf[b] = hv.nbuf[b] = 0;
    }
    const std::vector<RowState> none;
    e = enqueue_set(k, tab, none, st);
    if (e == cudaSuccess) e = enqueue_set(v, tab, none, st);
    if (e == cudaSuccess) e = scatter_rows(k, &stk, fr.data(), ft0.data(), fblk.data(), fs0.data(), nf, n_b, st);
    if (e == cudaSuccess) e = scatter_rows(v, &stv, fr.data(), ft0.data(), fblk.data(), fs0.data(), nf, n_b, st);
    if (e != cudaSuccess) return GEAR_ERR_CUDA;
  }
  // the new tokens, and every listed row's counters
  for (int i0 = 0; i0 < nrows && e == cudaSuccess; i0 += kAppendMax) {
    PagedAppend a;
    memset(&a, 0, sizeof(a));
    a.kbuf = k->buf;
    a.vbuf = v->buf;
    a.kn = k_new;
    a.vn = v_new;
    a.krows = k->rows;
    a.vrows = v->rows;
    a.B = k->B;
    a.H = k->H;
    a.n_b = n_b;
    a.n = nrows - i0 < kAppendMax ? nrows - i0 : kAppendMax;
    a.i0 = i0;
    for (int j = 0; j < a.n; ++j) {
      const int b = rows[i0 + j];
      a.row[j] = b;
      a.slot[j] = hk.nbuf[b];
      a.nblk[j] = hk.nblk[b];
      hk.nbuf[b] += 1;
      hv.nbuf[b] += 1;
    }
    e = paged_append_launch(a, esize(k->dtype), st);
  }
  update_maxima(k);
  update_maxima(v);
  return cuda_status(e);
}

gear_status gear_release_rows(gear_cache* c, const int32_t* rows, int32_t nrows, void* stream) {
  if (!paged_ok(c) || !rows_ok(c, rows, nrows)) return GEAR_ERR_INVALID_ARG;
  HostView h = host_view(c);
  std::vector<std::pair<int, int>> tab;
  std::vector<RowState> rs;
  for (int i = 0; i < nrows; ++i) {
    const int b = rows[i];
    for (int lp = 0; lp < c->pages_per_row; ++lp) {
      int32_t& e = h.table[(size_t)b * c->pages_per_row + lp];
      if (e < 0) continue;
      h.stack[(*h.top)++] = e;
      e = -1;
      tab.emplace_back(b * c->pages_per_row + lp, -1);
    }
    h.b0[b] = h.nblk[b] = h.nbuf[b] = 0;
    rs.push_back(RowState{b, 0, 0, 0});
  }
  update_maxima(c);
  return cuda_status(enqueue_set(c, tab, rs, (cudaStream_t)stream));
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
