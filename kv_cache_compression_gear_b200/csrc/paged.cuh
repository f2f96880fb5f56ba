// paged.cuh -- kernels of the paged cache layout: block-table and row-counter
// updates, buffer gathers, the scatter of a contiguous encode into pool pages
// and the per-row append. Argument blocks travel by value (kernel parameters),
// so the host needs no staging copies for them.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gear {

constexpr int kSetMax = 224;    // table entries per paged_set launch
constexpr int kSetRows = 32;    // row states per paged_set launch
constexpr int kRowsMax = 64;    // rows per gather / scatter launch
constexpr int kAppendMax = 128; // rows per append launch

// Table entries and row states to write (host-decided values).
struct PagedSet {
  int32_t* table;   // [B][ppr]
  int32_t* rows;    // [3][B]
  int32_t B;
  int32_t ntab, nrow;
  int32_t tab_idx[kSetMax], tab_val[kSetMax];
  int32_t row[kSetRows], b0[kSetRows], nblk[kSetRows], nbuf[kSetRows];
};

// Rows of one gather / scatter launch: entry i is batch row row[i], whose
// tokens land at row offset t0[i] as block blk[i] (per-channel key groups: its
// first token group at slot s0[i]); its units are unit (i0 + i) * H + h of the
// contiguous staging copy.
struct PagedRows {
  int32_t n, i0;
  int32_t row[kRowsMax], t0[kRowsMax], blk[kRowsMax], s0[kRowsMax];
};

// One tensor's staging copy (contiguous, one block) and its paged destination.
struct ScatterArgs {
  const uint8_t* s_codes;
  const uint8_t* s_meta;
  const uint8_t* s_oidx;
  const uint8_t* s_oval;
  const uint8_t* s_lfac;
  const float* s_rfac;
  uint8_t* d_codes;
  uint8_t* d_meta;
  uint8_t* d_oidx;
  uint8_t* d_oval;
  uint8_t* d_lfac;
  float* d_rfac;
  const int32_t* table;
  int32_t H, P, ppr, num_pages, nblk_max;
  int32_t nmax_s;                 // token rows per unit of the staging copy
  int32_t n;                      // tokens per unit
  int32_t wb, mb, kb, ob, lb;     // bytes per token: codes, meta, oidx, oval, lfac (mb = 0 with ch)
  int32_t rf_floats;              // Rf floats per unit and block (128 * r_pad)
  // per-channel key groups: meta is [unit][slot][128][2] floats; the block's
  // ceil(n / g) slots move from slot 0 of the staging unit to slot s0 of the row's unit
  int32_t ch, g, ch_slots_s, ch_slots_d;
};

// Per-row append: token i of k_new/v_new goes to buffer slot slot[i] of row
// row[i]; the row's counters become (blocks nblk[i], buffer fill slot[i] + 1).
struct PagedAppend {
  void* kbuf;
  void* vbuf;
  const void* kn;
  const void* vn;
  int32_t* krows;
  int32_t* vrows;
  int32_t B, H, n_b, n, i0;
  int32_t row[kAppendMax], slot[kAppendMax], nblk[kAppendMax];
};

cudaError_t paged_set_launch(const PagedSet& s, cudaStream_t st);
cudaError_t paged_gather_launch(const void* sk, const void* sv, void* dk, void* dv, int H, int unit_bytes,
                                const PagedRows& r, cudaStream_t st);
cudaError_t paged_scatter_launch(const ScatterArgs& s, const PagedRows& r, cudaStream_t st);
cudaError_t paged_append_launch(const PagedAppend& a, int esz, cudaStream_t st);

}  // namespace gear
