// kernels.h -- launch interface between the host planner and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "plan.h"

namespace rpa {

// The fused cache update is on in every product build.  A timing-only build
// of the library (compiled with RPA_ABLATE_CACHE_WRITE, into a separate file
// that nothing but the benchmark's --ablate-write leg loads) drops the stores
// of the new K/V rows, so that their cost inside the attention kernels can be
// measured; its caches are left unwritten and its results are not the
// method's.
#ifdef RPA_ABLATE_CACHE_WRITE
constexpr bool kCacheWrite = false;
#else
constexpr bool kCacheWrite = true;
#endif

// Device pointers and geometry shared by every kernel of one call.
struct Problem {
  const void *q;
  const void *k_new;
  const void *v_new;
  void *k_cache;
  void *v_cache;
  const int32_t *page_table;
  void *out;
  float *lse;          // may be null
  uint32_t *err;       // device error word (RPA_DEV_* bits)
  int32_t hq, hkv, d, p, num_pages, max_pages, dtype, causal;
  int32_t total_q;     // T: rows of q, k_new, v_new, out
  float scale;
  // Device-planned calls: the work counts (DeviceCount slots) written by the
  // planner kernel; each kernel takes min(its slot, the count it was launched
  // for).  nullptr: the launch counts are exact (host plan).
  const int32_t *dev_counts;
};

// Generic SIMT kernel: any dtype, any q_len, one warp per (row, query head).
cudaError_t launch_generic(const Problem &pb, const GenericSeq *seqs,
                           int n_seqs, int n_rows, cudaStream_t stream);

// Decode kernel (bf16): one CTA per (work item, KV head).
// partial_o: [n_partials, Hkv, G, D] fp32; partial_lse: [n_partials, Hkv, G].
// pack: four items per CTA, one per warp (short whole sequences).
cudaError_t launch_decode(const Problem &pb, const DecodeItem *items,
                          int n_items, float *partial_o, float *partial_lse,
                          bool pack, cudaStream_t stream);

// Split-KV combine: one warp per (combine item, query head).  pdl: queued
// with programmatic dependent launch right behind the decode launch it
// merges (its CTAs start during the decode tail and wait on the device).
cudaError_t launch_combine(const Problem &pb, const CombineItem *items,
                           int n_items, const float *partial_o,
                           const float *partial_lse, cudaStream_t stream, bool pdl);

// Small host-planned decode batches: the work items and combine rows travel
// in the kernels' launch parameters (host pointers), so no plan copy has to
// precede the kernels.  pdl: the combine is queued with programmatic
// dependent launch behind the decode launch.
bool decode_plan_fits_inline(int n_items, int n_combine);
cudaError_t launch_decode_inline(const Problem &pb, const DecodeItem *host_items,
                                 int n_items, float *partial_o, float *partial_lse,
                                 cudaStream_t stream);
cudaError_t launch_combine_inline(const Problem &pb, const CombineItem *host_rows,
                                  int n_items, const float *partial_o,
                                  const float *partial_lse, cudaStream_t stream, bool pdl);

// Prefill / chunked-prefill kernel (bf16, tcgen05): one CTA per (tile, query
// head).  head_dim 256: one 128-row tile per CTA.
cudaError_t launch_prefill(const Problem &pb, const PrefillTile *tiles,
                           int n_tiles, cudaStream_t stream);

// head_dim 64 / 128: two 128-row tiles per CTA (a 256-row work item);
// persistent, at most max_ctas CTAs (<= 0: one per SM).  split: K and V get
// a producer warp each (for context-heavy batches) instead of sharing one.
cudaError_t launch_prefill2(const Problem &pb, const PrefillTile *tiles,
                            int n_tiles, int max_ctas, bool split, cudaStream_t stream);

// head_dim 128 with a double-buffered score tile: persistent; pair: CTA
// pairs (clusters of two) sharing M = 256 MMAs, one 256-row work item per
// pair; otherwise one CTA per 128-row half of an item.  At most max_ctas
// CTAs (<= 0: as many as fit, one per SM).
cudaError_t launch_prefill3(const Problem &pb, const PrefillTile *tiles,
                            int n_tiles, int max_ctas, bool pair, cudaStream_t stream);

// Rows of a single prefill tile (query tokens per TMEM accumulator).
constexpr int kPrefillTileRows = 128;

// Rows of one prefill work item for a head dim.
// head_dim <= 128: 256 (two tiles, or a CTA pair); head_dim 256: 256 (a CTA
// pair), or 128 when RPA_OPT_PREFILL_KERNEL selects the one-tile kernel.
int prefill_item_rows(int head_dim);

}  // namespace rpa
