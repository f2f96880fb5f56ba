/*
 * gear.h -- C ABI of the GEAR KV-cache codec for NVIDIA B200 (sm_100a).
 *
 * GEAR compresses a KV-cache matrix X (tokens x head_dim) into three parts
 * (GEAR: Efficient KV Cache Compression for LLM Inference, Q3 on the method;
 * GEAR: An Efficient KV Cache Compression Recipe for Near-Lossless Generative
 * Inference of LLM, Abstract):
 *   S  - a sparse set holding the largest-magnitude entries exactly
 *        (S = Filter_s(X); Cites list, SqueezeLLM entry);
 *   D  - a uniform, group-wise, per-token b-bit quantization of the rest
 *        (Cites list, FlexGen entry);
 *   L.Rf^T - a rank-r approximation of the quantization residual, computed by
 *        power iteration (Q3, low-rank part; Cites list, PowerSGD entry),
 * so that X ~ D + L.Rf^T with the outlier slots overwritten by S.
 * New tokens go to a small full-precision streaming buffer that is compressed
 * when it fills (Q3, streaming strategy).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers (cudaMalloc'd or torch-owned)
 *    unless stated. The library never allocates device memory: caches and
 *    workspaces are carved from buffers the caller owns and sizes with the
 *    *_bytes() queries.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously on it. Argument validation runs on the
 *    host before any launch; on any status other than GEAR_ERR_CUDA nothing
 *    was enqueued. GEAR_ERR_CUDA means a launch or runtime call failed part
 *    way through; the caches the call was given are then undefined.
 *  - Element types: GEAR_F16 / GEAR_BF16 / GEAR_F32 for KV, queries, buffer
 *    and outlier values. Quantization metadata is fp32. Low-rank factors L are
 *    fp16 for 16-bit caches and fp32 for fp32 caches; Rf is always fp32.
 *  - Shapes are row-major, innermost dimension last, densely packed.
 *  - One "unit" is one (batch b, kv-head h) matrix; units are indexed
 *    u = b*H + h. Every unit of a contiguous cache holds the same number of
 *    tokens; a paged cache (gear_paged_cache_init) keeps counts per batch row.
 */
#ifndef GEAR_H_
#define GEAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GEAR_OK = 0,
  GEAR_ERR_INVALID_ARG = 1,  /* null pointer, bad shape/param, misalignment */
  GEAR_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. d != 128)   */
  GEAR_ERR_CAPACITY = 3,     /* would exceed n_max / nblk_max of the cache   */
  GEAR_ERR_CUDA = 4,         /* a CUDA runtime call failed                   */
  GEAR_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up           */
  GEAR_ERR_WORKSPACE = 6     /* workspace pointer null or too small          */
} gear_status;

typedef enum { GEAR_F16 = 0, GEAR_BF16 = 1, GEAR_F32 = 2 } gear_dtype;

/* Codec parameters -- the pages' statement of the problem.
 *  bits         b in {2, 4, 8}: code width of the quantized backbone
 *               (Q3: very low precision such as 4 bits).
 *  group_size   g: channels per quantization group; g divides d and g*b is a
 *               multiple of 32 (Cites: FlexGen entry, fine-grained grouping).
 *  outlier_frac s in [0, 0.5]: fraction of each token's entries kept exactly;
 *               k = ceil(s*d - 1e-9) outliers per token (Cites list,
 *               ZeroQuant entry: the paper fixes s at 2 %).
 *  rank         r in [0, 16], r <= min(n, d): rank of the residual factors of
 *               a block written by gear_encode (ZeroQuant entry: the paper
 *               uses 4 for prefill inputs).
 *  power_iters  T >= 1 when any rank > 0: power-iteration count, T counting
 *               (P, Q) update pairs (Cites list, PowerSGD entry).
 *  buffer_len   n_b >= 1: streaming-buffer length (Q3, streaming strategy).
 *  buffer_rank  r_buf in [0, 16], r_buf <= min(n_b, d): rank of each flushed
 *               buffer block (ZeroQuant entry: the paper gives every group of
 *               n_b decoded tokens rank 2).
 *  meta_f16     0: scale and zero point stored as fp32 (default); 1: stored as
 *               binary16, rounded to nearest even, with the codes decided
 *               against the stored values (a byte-lean layout: 4 instead of
 *               8 bytes per group; fp16 caches only, else UNSUPPORTED).
 *  channel_groups 0: the quantizer groups g channels of a token (default);
 *               1: the KIVI-combined key quantizer -- every channel gets its
 *               own (scale, zero) over each group of g consecutive tokens of a
 *               block (the last group of the block written by gear_encode may
 *               be shorter); outliers stay per token and are left out of the
 *               groups' min/max (GEAR: An Efficient KV Cache Compression
 *               Recipe ..., Cites list, KIVI entries: the buffer must be at
 *               least the group size; the same page's citing works, TailorKV
 *               entry: keys per channel, values per token). Requires a 16-bit
 *               cache, meta_f16 = 0, g in {32, 64, 128} and a buffer_len that
 *               is a multiple of g (>= g), so that every flushed buffer is
 *               whole groups (else INVALID_ARG / UNSUPPORTED). In decode such a
 *               cache serves as the K cache, with a V cache of channel_groups 0.
 *  seed         seeds the power-iteration start matrix Q0 (d x r): entry
 *               (i, j) is the (i*r + j)-th output of the splitmix64 stream
 *               whose state starts at `seed` (Steele, Lea & Flood, OOPSLA
 *               2014), top 24 bits mapped to [-1, 1) as u*2^-23 - 1. */
typedef struct gear_params {
  int32_t bits;
  int32_t group_size;
  float outlier_frac;
  int32_t rank;
  int32_t power_iters;
  int32_t buffer_len;
  int32_t buffer_rank;
  int32_t meta_f16;
  int32_t channel_groups;
  uint64_t seed;
} gear_params;

/* Compressed cache for ONE tensor (K or V) of one layer: B x H units, each with
 * up to n_max compressed tokens plus an n_b-token full-precision buffer.
 *
 * Filled by gear_cache_init(); the caller then treats it as opaque except for
 * reading the counters. n_max is stored rounded up to a multiple of 32 tokens. The struct lives in HOST memory; the arrays it points
 * to live in the caller's device buffer, laid out in this order, each array
 * starting on a 256-byte boundary:
 *
 *   codes  uint32 [U][n_max][W]      W = d*b/32. Channel c of a token is bits
 *                                    [(c*b)%32, (c*b)%32 + b) of word c*b/32.
 *   meta   float  [U][n_max][G][2]   G = d/g; (scale, zero) of each group,
 *                                    zero = group minimum over non-outliers
 *                                    (binary16 [U][n_max][G][2] if meta_f16).
 *                                    With channel_groups: float
 *                                    [U][S][d][2], S = ceil(n_max/g) + 1 token
 *                                    groups; token t of block 0 is in group
 *                                    t / g, token t of a flushed block in group
 *                                    ceil(blk0_len/g) + (t - blk0_len) / g.
 *   oidx   uint8  [U][n_max][k]      outlier channels, ascending.
 *   oval   dtype  [U][n_max][k]      outlier values, bit-exact input copies.
 *   lfac   f16|f32[U][n_max][r_max]  L rows, stored as L * 2^e_blk.
 *   rfac   float  [U][nblk_max][d][r_pad]  Rf rows (one per channel), stored as
 *                                    Rf * 2^-e_blk; r_pad = r_max rounded up
 *                                    to a multiple of 4, the padding zero.
 *   buf    dtype  [U][n_b][d]        streaming buffer (full precision).
 *
 * with U = B*H, k = outliers per token, r_max = max(rank, buffer_rank) and
 * e_blk = floor(log2(block_len) / 2) (the factor keeps fp16 L rows near unit
 * magnitude; L * Rf^T is unchanged). Blocks: block 0 holds tokens
 * [0, blk0_len) with rank blk0_rank; block i >= 1 holds the n_b tokens
 * [blk0_len + (i-1)*n_b, blk0_len + i*n_b) with rank buffer_rank. */
typedef struct gear_cache {
  /* geometry and parameters (written by gear_cache_init) */
  int32_t B, H, d, n_max, nblk_max;
  int32_t dtype;      /* gear_dtype */
  gear_params p;
  int32_t k, G, W, r_max;
  /* device arrays carved from the caller's buffer (not owned) */
  uint32_t* codes;
  float* meta;
  uint8_t* oidx;
  void* oval;
  void* lfac;
  float* rfac;
  void* buf;
  /* host-side counters, advanced by gear_encode / gear_append_buffer */
  int32_t n_comp;     /* compressed tokens per unit                  */
  int32_t n_buf;      /* tokens currently in the streaming buffer    */
  int32_t n_blk;      /* compressed blocks                           */
  int32_t blk0_len;   /* tokens in block 0 (0 while n_blk == 0)      */
  int32_t blk0_rank;  /* rank of block 0                             */
  int32_t reserved1;
  /* paged layout (gear_paged_cache_init); all zero for a contiguous cache */
  int32_t page_tokens;    /* P: tokens per page, a multiple of 32         */
  int32_t num_pages;      /* pages in the pool                            */
  int32_t pages_per_row;  /* block-table row length                       */
  int32_t reserved2;
  int32_t* table;         /* device [B][pages_per_row] pool page of each logical page, -1 if none */
  int32_t* rows;          /* device [3][B] per row: block-0 length, blocks, buffer fill */
  int32_t* host;          /* host, caller-owned: see gear_paged_host_ints  */
} gear_cache;

/* Number of outliers kept per token: k = ceil(s*d - 1e-9), computed in double
 * (so s = 2% at d = 128 keeps 3 entries, s = 5% keeps 7). */
int32_t gear_num_outliers(float outlier_frac, int32_t d);

/* Checks a parameter set (the limits listed at gear_params). */
gear_status gear_validate_params(const gear_params* p, int32_t d);

/* Bytes of device memory a cache with this geometry needs (0 on bad args). */
size_t gear_cache_bytes(const gear_params* p, int32_t B, int32_t H, int32_t d,
                        int32_t n_max, int32_t nblk_max, gear_dtype dtype);

/* Lays a cache out in [dev, dev + bytes). `dev` must be 256-byte aligned and
 * bytes >= gear_cache_bytes(...). Sets counters to zero. Writes no device
 * memory. Errors: INVALID_ARG (null, misaligned, bad params), UNSUPPORTED
 * (d != 128), CAPACITY (bytes too small). */
gear_status gear_cache_init(gear_cache* c, const gear_params* p, int32_t B, int32_t H,
                            int32_t d, int32_t n_max, int32_t nblk_max, gear_dtype dtype,
                            void* dev, size_t bytes);

/* Empties a cache for reuse with the same geometry and parameters: sets the
 * counters (n_comp, n_buf, n_blk, blk0_len, blk0_rank) to zero, so that the
 * next gear_encode writes block 0 again. Host bookkeeping only: writes no device
 * memory and enqueues nothing (the old contents are simply overwritten by the
 * next encode and appends). Errors: INVALID_ARG (null). */
gear_status gear_cache_reset(gear_cache* c);

/* Workspace bytes gear_encode needs to encode n tokens per unit of c. */
size_t gear_encode_workspace_bytes(const gear_cache* c, int32_t n);

/* Encodes kv [B][H][n][d] (cache dtype, 16-byte aligned) as block 0 of an empty
 * cache, with rank p.rank: outliers, per-token group-wise quantization and the
 * rank-r power-iteration factors of the residual (Q3; Cites: SqueezeLLM,
 * FlexGen and PowerSGD entries). Requires c->n_comp == 0 and n_buf == 0,
 * 1 <= n <= n_max, rank <= n. On success sets n_comp = n, n_blk = 1.
 * Errors: INVALID_ARG, CAPACITY, WORKSPACE, CUDA. */
gear_status gear_encode(gear_cache* c, const void* kv, int32_t n,
                        void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes gear_encode_batch needs for `count` caches shaped like
 * caches[0] (host array), n tokens per unit. */
size_t gear_encode_batch_workspace_bytes(int32_t count, const gear_cache* const* caches, int32_t n);

/* gear_encode of kv[i] into caches[i] for every i < count, with up to 16
 * tensors (the K and V of a layer, the layers of a model) sharing each kernel
 * launch. The pages have no counterpart: it only batches the per-tensor
 * encode. caches and kv are HOST arrays of `count` pointers; the caches must
 * be distinct, empty and alike in B, H, dtype, n_max, nblk_max and params.
 * Codes, meta and outliers are bit-identical to gear_encode's; L and Rf may
 * differ in the last bits (the Gram partials are grouped by the launch's
 * tiling). Larger batches run as consecutive launches on the stream.
 * Errors: INVALID_ARG, CAPACITY, UNSUPPORTED, WORKSPACE, CUDA. */
gear_status gear_encode_batch(int32_t count, gear_cache* const* caches, const void* const* kv, int32_t n,
                              void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes gear_decode_attn needs for these caches and Hq query heads. */
size_t gear_decode_workspace_bytes(const gear_cache* k, const gear_cache* v, int32_t Hq);

/* One decode step of attention over the compressed caches plus buffers:
 *   out[b][j] = sum_t softmax_t(scale * q[b][j] . Khat[b][h][t]) Vhat[b][h][t]
 * over the n_comp compressed tokens (Khat/Vhat = dequantized codes + L.Rf^T,
 * outlier slots replaced by their exact values) followed by the n_buf buffer
 * tokens, with h = j / (Hq / H) (grouped-query sharing).
 *   q    [B][Hq][d], cache dtype.       out  [B][Hq][d], out_dtype
 *   out_dtype is the cache dtype or GEAR_F32.
 * k and v must have identical geometry, counters and parameters, except that
 * k may have channel_groups = 1 where v has 0; Hq % H == 0.
 * Errors: INVALID_ARG, WORKSPACE, CUDA. */
gear_status gear_decode_attn(const gear_cache* k, const gear_cache* v, const void* q,
                             int32_t Hq, float softmax_scale, void* out, gear_dtype out_dtype,
                             void* workspace, size_t ws_bytes, void* stream);

/* Decode attention over a batch whose prefills were right-padded to one length
 * (serving with sequences of different prompt lengths; no counterpart in the
 * paper, which decodes one batch of equal lengths). Same computation, layouts
 * and errors as gear_decode_attn, except that for batch row b the block-0
 * tokens [prefill_len[b], blk0_len) are padding and take no part in the
 * softmax; every later token (flushed blocks and buffer) is real.
 *   prefill_len  [B] int32 in DEVICE memory, read by the kernel; values are
 *                clamped to [0, blk0_len]. Block 0 is the block gear_encode wrote.
 * A row of q whose every token is padding gets an output of 0.
 * Errors: INVALID_ARG (also for a null or unaligned prefill_len), WORKSPACE, CUDA. */
gear_status gear_decode_attn_ragged(const gear_cache* k, const gear_cache* v, const void* q, int32_t Hq,
                                    float softmax_scale, void* out, gear_dtype out_dtype,
                                    const int32_t* prefill_len, void* workspace, size_t ws_bytes,
                                    void* stream);

/* Decode attention that allocates nothing. The GEAR paper has no counterpart
 * of this entry point: it exists for callers that cannot call cudaMalloc or
 * hand the library a workspace -- for example a plugin inside a host framework
 * that owns all device memory and offers plugins no allocator, or a decode loop
 * whose device memory budget is fixed when the process starts.
 * Same computation, arguments, layouts and errors as gear_decode_attn, except
 * that the split-K partial results go to a scratch array inside the library: a
 * file-scope __device__ array of 4 MiB that every GPU which loads the library
 * holds until the process exits. The caller still passes q and out.
 * Limit: returns GEAR_ERR_WORKSPACE, enqueuing nothing, when the partials would
 * not fit, i.e. when gear_decode_workspace_bytes(k, v, Hq) > 4 MiB (each of the
 * B * Hq query rows needs 520 bytes per split). The number of splits follows
 * from the device's SM count (the split-K grid is one wave of resident warps),
 * so whether a problem fits depends on the device: a caller that must know in
 * advance checks gear_decode_workspace_bytes(k, v, Hq) <= 4 MiB with the target
 * device current.
 * Set-up: the first call on a device looks up the array's device address with
 * cudaGetSymbolAddress and caches it; make that first call before any stream
 * capture. All calls share the one array and it keeps the last call's contents:
 * calls that overlap on the GPU (different streams, or threads) race and
 * corrupt each other's results, so serialize them. Every call writes each
 * scratch entry before reading it, so nothing needs clearing. */
gear_status gear_decode_attn_noalloc(const gear_cache* k, const gear_cache* v, const void* q, int32_t Hq,
                                     float softmax_scale, void* out, gear_dtype out_dtype, void* stream);

/* Workspace bytes gear_append_buffer needs (covers the flush encode). */
size_t gear_append_workspace_bytes(const gear_cache* k);

/* Appends one token per unit, k_new/v_new [B][H][d] (cache dtype). If the
 * buffer already holds n_b tokens, they are first compressed as a new block
 * of rank buffer_rank (same codec as gear_encode) appended after the
 * compressed tokens, and the buffer is emptied (Q3, streaming strategy: the
 * buffer is compressed once it is full). Then the new token is
 * written to buffer slot n_buf. Errors: INVALID_ARG, CAPACITY, WORKSPACE, CUDA. */
gear_status gear_append_buffer(gear_cache* k, gear_cache* v, const void* k_new,
                               const void* v_new, void* workspace, size_t ws_bytes,
                               void* stream);

/* Debug/test export: writes the reconstruction of every token of c,
 * out_f32 [B][H][n_comp + n_buf][d] fp32 (compressed tokens first, then the
 * buffer). Errors: INVALID_ARG, CUDA. */
gear_status gear_decode_dense(const gear_cache* c, float* out_f32, void* stream);

/* ------------------------------------------------------------ paged layout
 * Serving integration (GEAR: Efficient KV Cache Compression for LLM Inference,
 * Q5 on integration into real-time inference systems; the pages give no
 * layout, so this one is the library's own). In a paged cache every batch row
 * b (one sequence: its H units) has its own counters -- block-0 length, number
 * of blocks, buffer fill -- so that rows join (gear_encode_rows), grow
 * (gear_append_rows, flushing each row's buffer when that row's buffer is
 * full) and leave (gear_release_rows) independently. The per-token arrays
 * (codes, meta, oidx, oval, lfac) live in a pool of num_pages pages of P
 * tokens; a row's compressed tokens are numbered from 0 as in a contiguous
 * cache (block 0, then n_b per flushed block) and token t of row b, head h is
 * pool row (table[b][t / P] * H + h) * P + t % P. The library hands pages out
 * from the pool as rows grow and takes them back on release. Per-token arrays
 * are laid out as in a contiguous cache with [U][n_max] replaced by
 * [num_pages][H][P]; rfac [U][nblk_max][d][r_pad] and buf [U][n_b][d] stay per
 * unit; then table [B][pages_per_row] and rows [3][B] (int32).
 * The cache-level counters n_comp, n_buf and n_blk hold the maxima over rows;
 * blk0_len is 0 (per row) and blk0_rank is p.rank.
 * gear_decode_attn, gear_decode_attn_ragged and gear_decode_attn_noalloc take
 * paged caches (both K and V paged, built by the same calls on the same rows,
 * so that their counters and tables agree; INVALID_ARG otherwise): each row
 * attends over its own tokens, a row without tokens gets an output of 0.
 * The decode work split runs over the tokens the rows hold (rows laid end to
 * end at their own lengths), so a ragged batch costs what its tokens cost.
 * gear_encode, gear_encode_batch, gear_append_buffer,
 * gear_cache_reset and gear_decode_dense return UNSUPPORTED on a paged cache.
 * Per-channel key groups (channel_groups = 1, a K cache of 16-bit values): the
 * meta slots stay per unit, [U][S][d][2] fp32 with S = ceil(P * pages_per_row /
 * g) + 1, numbered per row as in a contiguous cache with that row's block-0
 * length; the V cache beside it has channel_groups = 0.
 * Limits: P a multiple of 32 (a decode tile of 32 tokens never spans two pages). */

/* Host int32 entries a paged cache keeps in caller memory:
 * 3*B counters (block-0 length, blocks, buffer fill per row), the table
 * mirror [B][pages_per_row], a stack of free pages [num_pages] and its
 * height (1). The host array must stay alive and untouched while the cache
 * is used. */
size_t gear_paged_host_ints(int32_t B, int32_t pages_per_row, int32_t num_pages);

/* Device bytes of a paged cache (0 on bad args). A row holds at most
 * page_tokens * pages_per_row compressed tokens and nblk_max blocks. */
size_t gear_paged_cache_bytes(const gear_params* p, int32_t B, int32_t H, int32_t d, int32_t page_tokens,
                              int32_t num_pages, int32_t pages_per_row, int32_t nblk_max, gear_dtype dtype);

/* Lays a paged cache out in [dev, dev + bytes) (256-byte aligned) with host
 * state in host[0 .. host_ints). Every row starts empty and every page free.
 * Enqueues two memsets on `stream` (counters to 0, table to -1).
 * Errors: INVALID_ARG (null, misaligned, bad geometry, P % 32 != 0),
 * UNSUPPORTED (d != 128, pool rows >= 2^31, per-channel key groups of fp32),
 * CAPACITY (bytes or host_ints too small), CUDA. */
gear_status gear_paged_cache_init(gear_cache* c, const gear_params* p, int32_t B, int32_t H, int32_t d,
                                  int32_t page_tokens, int32_t num_pages, int32_t pages_per_row, int32_t nblk_max,
                                  gear_dtype dtype, void* dev, size_t bytes, int32_t* host, size_t host_ints,
                                  void* stream);

/* Workspace bytes gear_encode_rows needs for nrows rows of n tokens. */
size_t gear_encode_rows_workspace_bytes(const gear_cache* c, int32_t nrows, int32_t n);

/* Encodes kv [nrows][H][n][d] (cache dtype, 16-byte aligned) as block 0 of
 * the empty rows rows[0 .. nrows) (HOST array of distinct row indices), with
 * rank p.rank -- the computation of gear_encode, row by row. Takes
 * ceil(n / P) pages per row from the pool. The codec runs on a contiguous
 * copy in the workspace, which a scatter kernel then moves into the pages.
 * Errors: INVALID_ARG (not paged, bad or repeated row, row not empty,
 * rank > n), CAPACITY (n > P * pages_per_row, too few free pages),
 * WORKSPACE, CUDA. */
gear_status gear_encode_rows(gear_cache* c, const int32_t* rows, int32_t nrows, const void* kv, int32_t n,
                             void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes gear_append_rows needs (covers a flush of every row). */
size_t gear_append_rows_workspace_bytes(const gear_cache* k);

/* Appends one token to each of the rows rows[0 .. nrows) (HOST array of
 * distinct, already encoded rows): k_new/v_new [nrows][H][d], cache dtype.
 * A listed row whose buffer holds n_b tokens is flushed first: its buffer is
 * compressed as that row's next block with rank buffer_rank and the buffer
 * emptied (Q3, streaming strategy, row by row), taking pages from the pool as
 * needed. Rows not listed are left as they are.
 * Errors: INVALID_ARG (caches not a matching paged pair, bad, repeated or
 * unencoded row), CAPACITY (a flush past P * pages_per_row tokens or nblk_max
 * blocks, too few free pages), WORKSPACE, CUDA. */
gear_status gear_append_rows(gear_cache* k, gear_cache* v, const int32_t* rows, int32_t nrows, const void* k_new,
                             const void* v_new, void* workspace, size_t ws_bytes, void* stream);

/* Empties the rows rows[0 .. nrows) (HOST array) and returns their pages to
 * the pool; the rows can then be encoded again. Enqueues the counter and
 * table updates on `stream`. Errors: INVALID_ARG, CUDA. */
gear_status gear_release_rows(gear_cache* c, const int32_t* rows, int32_t nrows, void* stream);

/* Reads (host, synchronous) and clears the device-side error word that
 * kernels set instead of trapping (GEAR_ERR_* value, 0 if none). */
gear_status gear_get_device_status(int32_t* status);

/* Failure-detection self-test (no counterpart in the paper): launches one warp
 * that waits on an mbarrier nothing ever completes, bounded by limit_us
 * microseconds (1 .. 1000000) of wall time. The bound runs out, the kernel
 * records GEAR_ERR_TIMEOUT in the device error word and returns; nothing
 * traps, and the context stays usable. Asynchronous on `stream`; read the
 * result with gear_get_device_status after synchronizing.
 * Errors: INVALID_ARG (limit out of range), CUDA. */
gear_status gear_selftest_wait_timeout(uint32_t limit_us, void* stream);

/* Static description of a status code. */
const char* gear_status_string(gear_status s);

/* Library version as "major.minor.patch". */
const char* gear_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GEAR_H_ */
