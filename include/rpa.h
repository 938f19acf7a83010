/*
 * rpa.h -- C ABI of librpa_b200.so: ragged paged attention on NVIDIA B200
 * (sm_100a).
 *
 * The operation ("Ragged Paged Attention: A High-Performance and Flexible LLM
 * Inference Kernel for TPU", arXiv 2604.15464, abstract): one attention pass
 * over a ragged batch whose sequences may be decoding (one new token),
 * prefilling (every token new) or both (new tokens after a cached context),
 * where each sequence's keys and values live in fixed-size pages of a shared
 * pool addressed through a per-sequence page table (RPA talk summary,
 * rocketrecap.com, glossary "PagedAttention"), and where the new tokens' K/V
 * are written into their cache pages by the same kernels that attend over
 * them (talk summary 00:06:36).  Attention is exact softmax attention
 * (glossary "FlashAttention"); the result does not depend on how the batch
 * is split across kernels.
 *
 * Notation: S sequences; sequence s has q_len[s] = cu_q_lens[s+1] -
 * cu_q_lens[s] new tokens and kv_len[s] >= q_len[s] tokens in total, so its
 * first c[s] = kv_len[s] - q_len[s] tokens are already cached.  T =
 * cu_q_lens[S] new tokens in all.  Hq query heads, Hkv KV heads, G = Hq/Hkv;
 * query head h reads KV head h / G.  D = head_dim, P = page_size.
 *
 * All functions are thread-safe, never throw, never abort and never free
 * memory they did not allocate.
 */
#ifndef RPA_H
#define RPA_H

#include <stdint.h>

#if defined(__GNUC__)
#define RPA_API __attribute__((visibility("default")))
#else
#define RPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of q, k_new, v_new, the caches and out (all the same). */
typedef enum { RPA_F32 = 0, RPA_BF16 = 1 } rpa_dtype;

/* Return codes. */
enum {
  RPA_OK = 0,
  RPA_ERR_INVALID_ARG = 1,   /* null pointer where one is required, bad dims */
  RPA_ERR_UNSUPPORTED = 2,   /* head_dim not in {64,128,256}; page_size not a
                                power of two in [8,256]; Hq % Hkv != 0; G > 16 */
  RPA_ERR_LENGTHS = 3,       /* cu_q_lens not starting at 0 / decreasing;
                                kv_len < q_len; more pages than
                                max_pages_per_seq; T != total_q_tokens */
  RPA_ERR_DISTRIBUTION = 4,  /* distribution given and inconsistent */
  RPA_ERR_OOM = 5,           /* library workspace could not be allocated */
  RPA_ERR_CUDA = 6,          /* a CUDA call or kernel launch failed */
  RPA_ERR_SCRATCH_LIMIT = 7, /* rpa_decode_noalloc: the batch needs more
                                scratch than its fixed array holds */
  RPA_ERR_WORKSPACE = 8      /* rpa_forward_device: the caller's workspace
                                is smaller than rpa_device_workspace_size
                                reports or not 256-byte aligned */
};

/* Bits of the device error word read by rpa_device_status(). */
#define RPA_DEV_BAD_PAGE 0x1u /* a page-table entry outside [0, num_pages)
                                 was met; that page was read as zeros and
                                 nothing was written to it */
#define RPA_DEV_TIMEOUT 0x2u  /* a bounded wait on a shared-memory barrier ran
                                 out; the CTA stopped early, outputs of that
                                 CTA are incomplete */
#define RPA_DEV_BAD_LENGTHS 0x4u /* rpa_forward_device: the device-resident
                                 lengths broke a rule rpa_forward checks on the
                                 host (RPA_ERR_LENGTHS) or num_seqs was
                                 outside [0, max_seqs]; the call did nothing
                                 else: no cache slot, out or lse row was
                                 written */

/* Problem geometry. */
typedef struct {
  int32_t num_q_heads;       /* Hq */
  int32_t num_kv_heads;      /* Hkv, divides Hq */
  int32_t head_dim;          /* D: 64, 128 or 256 */
  int32_t page_size;         /* P: power of two, 8..256 */
  int32_t num_pages;         /* physical pages in each cache */
  int32_t max_pages_per_seq; /* row length of page_table */
  int32_t total_q_tokens;    /* T, must equal cu_q_lens[num_seqs] */
  int32_t dtype;             /* rpa_dtype */
} rpa_dims;

/*
 * rpa_forward -- one ragged paged attention pass.
 *
 * Device buffers (row-major, contiguous, all of dims->dtype unless noted):
 *   q        [T, Hq, D]       read
 *   k_new    [T, Hkv, D]      read: K of the new tokens, in token order
 *   v_new    [T, Hkv, D]      read
 *   k_cache  [num_pages, P, Hkv, D]  read and written in place
 *   v_cache  [num_pages, P, Hkv, D]  read and written in place
 *   page_table [num_seqs, max_pages_per_seq] int32: logical page j of
 *            sequence s is physical page page_table[s][j]; only the first
 *            ceil(kv_len[s] / P) entries of a row are read
 *   out      [T, Hq, D]       written for every row
 *   lse      [T, Hq] float32  written for every row, or NULL
 * Host buffers:
 *   cu_q_lens [num_seqs + 1] int32, cu_q_lens[0] = 0, non-decreasing
 *   kv_lens   [num_seqs] int32, kv_len[s] >= q_len[s]
 *   distribution [3] int32 or NULL: cumulative counts {d, p, S}.  Sequences
 *            [0, d) are decode (q_len <= 1), [d, p) fresh prefill
 *            (q_len == kv_len), [p, S) mixed / chunked prefill (any q_len <=
 *            kv_len).  This is the pages' distribution-aware split into
 *            decode, prefill and mixed work (arXiv 2604.15464, abstract,
 *            technique 3).  NULL: the library classifies each sequence
 *            itself and sequence order does not matter.  It only chooses
 *            kernels; results never depend on it.
 * scale: the factor on q.k (1/sqrt(D) for standard attention); it must be
 *            positive and finite, otherwise RPA_ERR_INVALID_ARG.
 *
 * Semantics (exact attention; talk summary 00:06:36 for the order):
 *   1. for every s and i < q_len[s], K/V of new token cu_q_lens[s] + i are
 *      copied bit for bit into slot (c[s] + i) % P of physical page
 *      page_table[s][(c[s] + i) / P] of k_cache / v_cache;
 *   2. query row t = cu_q_lens[s] + i, head h attends over positions
 *      j < kv_len[s] of the updated cache with KV head h / G, restricted to
 *      j <= c[s] + i when causal != 0 (the mask is aligned to the end of the
 *      sequence): out = sum_j softmax_j(scale * q.k_j) v_j, accumulated in
 *      fp32 and rounded to nearest-even into dtype;
 *      lse = ln sum_j exp(scale * q.k_j) over the same positions (fp32).
 *   Cache slots other than those of step 1 are never written; slots past
 *   kv_len and unused pages are never read (they may hold NaN).
 *
 * Ownership and aliasing: the caller owns every buffer.  out and lse must
 * not overlap any input.  Pages written by one call must not be shared by
 * two sequences of that call.  The library keeps a per-device workspace
 * (descriptor buffers, split-KV partials, the error word) that it grows on
 * demand and frees at process exit.
 *
 * stream: a cudaStream_t (NULL = legacy default stream).  The call is
 * asynchronous: it validates and plans on the host, queues one small
 * host-to-device copy of the plan and the kernels on `stream`, and returns.
 * num_seqs == 0 or T == 0 with no kv work is a successful no-op.
 *
 * Returns RPA_OK or an RPA_ERR_* code; on an error nothing was queued and no
 * buffer was touched.  Device-side conditions are reported through
 * rpa_device_status().
 */
RPA_API int rpa_forward(const void *q, const void *k_new, const void *v_new,
                void *k_cache, void *v_cache, const int32_t *page_table,
                const int32_t *cu_q_lens, const int32_t *kv_lens,
                int32_t num_seqs, const int32_t *distribution, float scale,
                int32_t causal, void *out, float *lse, const rpa_dims *dims,
                void *stream);

/*
 * rpa_device_status -- synchronise `stream`, then read and clear the current
 * device's error word (RPA_DEV_* bits, 0 when nothing happened) into *flags.
 * Returns RPA_OK, or RPA_ERR_CUDA if the synchronisation reported an error.
 */
RPA_API int rpa_device_status(void *stream, uint32_t *flags);

/* Static, human-readable name of a return code. */
RPA_API const char *rpa_status_string(int status);

/* What the host planner made of a batch (host only, no GPU needed). */
typedef struct {
  int32_t num_decode;        /* sequences run by the decode kernel */
  int32_t num_prefill;       /* sequences run by the prefill kernel */
  int32_t num_generic;       /* sequences run by the generic kernel */
  int32_t num_empty;         /* q_len == 0 sequences */
  int32_t decode_items;      /* (sequence, kv chunk) work items, per KV head */
  int32_t decode_max_splits; /* most chunks any one decode sequence got */
  int32_t combine_rows;      /* decode sequences that need the LSE combine */
  int32_t prefill_tiles;     /* (sequence, query tile) work items, per Q head */
  int64_t plan_bytes;        /* bytes of the plan copied to the device */
  int32_t decode_packed;     /* of decode_items: short whole sequences run
                                four per CTA, one per warp */
  int32_t pad;
} rpa_plan_info;

/*
 * rpa_plan -- run validation and the host planner exactly as rpa_forward
 * would for these lengths and dims, without touching any device.  Returns
 * the same RPA_ERR_* codes rpa_forward would; fills *info on RPA_OK.
 */
RPA_API int rpa_plan(const int32_t *cu_q_lens, const int32_t *kv_lens,
             int32_t num_seqs, const int32_t *distribution,
             const rpa_dims *dims, rpa_plan_info *info);

/* Planner knobs (process-wide).  Each returns the previous value. */
enum {
  RPA_OPT_DECODE_CHUNK_BLOCKS = 0, /* 16-token blocks per decode work item
                                      (default 192; <= 0 restores it) */
  RPA_OPT_FORCE_GENERIC = 1,       /* 1: run every sequence on the generic
                                      kernel (default 0) */
  RPA_OPT_DISABLE_PREFILL_TC = 2,  /* 1: prefill sequences use the generic
                                      kernel instead of tensor cores */
  RPA_OPT_PREFILL_SMS = 3,         /* SMs of the prefill kernel in a
                                      concurrent mixed batch: k > 0 at most
                                      k; 0 (default) sized from the plan, the
                                      prefill's estimated share of the two
                                      kernels' SM-time (x1.2, even, at least
                                      16; rpa_forward_device: every SM);
                                      < 0 every SM */
  RPA_OPT_CONCURRENT_MIXED = 4,    /* >= 0 (default 0): the prefill and the
                                      decode work of a mixed batch run
                                      concurrently, prefill on a
                                      highest-priority library stream that the
                                      caller's stream joins before the call
                                      returns (rpa_forward_host: its groups
                                      with prefill rows likewise); < 0: one
                                      after the other */
  RPA_OPT_PREFILL_LOADERS = 5,     /* TMA producer warps of the head_dim <= 128
                                      prefill kernel: 1 (K and V share one), 2
                                      (one each; the cache update gets one warp
                                      instead of two), 0 = chosen per batch:
                                      2 when the prefill rows' cached context
                                      outnumbers their new tokens (default 0) */
  RPA_OPT_DECODE_PACK_BLOCKS = 6,  /* decode sequences of at most this many
                                      16-token blocks (and within one work
                                      item) run four per CTA, one per warp,
                                      when they make at least 296 such CTAs
                                      (two per SM); fewer stay in the main
                                      decode launch (default 64; 0 restores
                                      it, < 0: never) */
  RPA_OPT_PREFILL_KERNEL = 7       /* prefill kernel.  0 (default): the
                                      head_dim 64 / 128 kernel with two
                                      128-row tiles per CTA, and CTA pairs
                                      sharing M = 256 tcgen05 MMAs at
                                      head_dim 256 (one 256-row item per
                                      pair); 1: the two-tile kernel, and one
                                      128-row tile per CTA at head_dim 256;
                                      2: CTA pairs at head_dim 128 and 256;
                                      3: the head_dim 128 pair design on one
                                      CTA per 128-row tile.  Results agree
                                      within rounding.  The device workspace
                                      size depends on it at head_dim 256
                                      (item rows) */
};
RPA_API int64_t rpa_set_option(int32_t option, int64_t value);

/* Kernel classes reported by rpa_profile_read(). */
enum { RPA_KERNEL_GENERIC = 0, RPA_KERNEL_DECODE = 1, RPA_KERNEL_COMBINE = 2,
       RPA_KERNEL_PREFILL = 3, RPA_KERNEL_CLASSES = 4 };

/*
 * rpa_profile_enable -- tracing switch (process-wide, default off).  While
 * on, every kernel launch of rpa_forward and rpa_forward_host is bracketed
 * by two CUDA events on the launching stream (rpa_forward_device and
 * rpa_decode_noalloc are not traced).  The records accumulate until
 * rpa_profile_read collects them, so a long traced run should read them
 * from time to time.  Returns the previous setting.
 */
RPA_API int32_t rpa_profile_enable(int32_t on);

/*
 * rpa_profile_read -- wait for every traced launch, add up their device
 * durations per kernel class and forget them.  ms[RPA_KERNEL_CLASSES]
 * receives milliseconds, launches[RPA_KERNEL_CLASSES] launch counts (either
 * may be NULL).  Returns RPA_OK or RPA_ERR_CUDA.
 */
RPA_API int rpa_profile_read(double *ms, int64_t *launches);

/*
 * rpa_decode_noalloc -- decode-only variant of rpa_forward that allocates
 * nothing.  The pages have no counterpart to this entry point: it exists for
 * callers that cannot call cudaMalloc at the point where they run attention
 * (a memory pool or allocator servicing a request, a serving process whose
 * device memory is fully reserved up front, a hard memory budget), because
 * rpa_forward grows a per-device workspace on demand.
 *
 * Every sequence has exactly one new token: token s belongs to sequence s,
 * dims->total_q_tokens == num_seqs, kv_lens[s] >= 1 (host), dtype bf16.
 * Buffers, layouts and results are those of rpa_forward for such a batch
 * (causal and non-causal coincide for one new token); the new K/V are
 * stored into the cache by the same kernels.  dev_flags: device uint32 that
 * receives RPA_DEV_* bits (OR-ed in, never cleared), or NULL to discard them.
 *
 * Scratch: all plan and split-KV buffers live in one file-scope device array
 * of 16 MiB that every GPU loading this part of the library holds until the
 * process exits.  A batch whose work items, combine rows or partial results
 * do not fit is rejected with RPA_ERR_SCRATCH_LIMIT before any device work
 * (8192 work items of at most RPA_OPT_DECODE_CHUNK_BLOCKS 16-token blocks,
 * 192 by default; partial results of
 * num_kv_heads * G * (head_dim + 1) floats per split item within ~15.6 MiB).
 * No cudaMalloc, cudaFree, cudaMallocHost or other allocating routine is
 * called.  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and creates one event, with that device current;
 * make that first call before any stream capture.  All calls share the one
 * array and it keeps the last call's contents: calls that can overlap on the
 * GPU race on it, so the caller must order them (for example, one stream per
 * device).
 *
 * The plan is staged in static host arrays and copied with cudaMemcpyAsync;
 * an event recorded after those copies is waited for by the next call before
 * it rewrites the arrays, so a call may block until the previous call's plan
 * copy has run on its stream.  A call on a stream that is being captured
 * into a CUDA graph returns RPA_ERR_INVALID_ARG before any device work (its
 * plan would be read from arrays that later calls rewrite).
 */
RPA_API int rpa_decode_noalloc(const void *q, const void *k_new,
                               const void *v_new, void *k_cache,
                               void *v_cache, const int32_t *page_table,
                               const int32_t *kv_lens, int32_t num_seqs,
                               float scale, void *out, float *lse,
                               const rpa_dims *dims, uint32_t *dev_flags,
                               void *stream);

/*
 * rpa_device_workspace_size -- bytes of device workspace rpa_forward_device
 * needs for batches of at most max_seqs sequences under dims (total_q_tokens
 * is the row capacity T of q / k_new / v_new / out).  It depends on dims,
 * max_seqs and the current RPA_OPT_DECODE_CHUNK_BLOCKS and
 * RPA_OPT_DECODE_PACK_BLOCKS values (and, at head_dim 256,
 * RPA_OPT_PREFILL_KERNEL) only.  Host only; returns RPA_OK or the
 * RPA_ERR_* code of bad dims / max_seqs < 0 (then *bytes = 0).
 */
RPA_API int rpa_device_workspace_size(const rpa_dims *dims, int32_t max_seqs,
                                      int64_t *bytes);

/*
 * rpa_forward_device -- rpa_forward with the metadata pass on the GPU, for
 * CUDA-graph capture.  The pages propose moving the kernel's scalar metadata
 * work off the main compute path (talk summary 00:16:06 and 00:18:14: SparseCore
 * offload); here a one-CTA planner kernel, queued on `stream` before the
 * attention kernels, reads the lengths from device memory and writes the
 * work lists into `workspace`.
 *
 * Differences from rpa_forward:
 *   cu_q_lens [max_seqs + 1], kv_lens [max_seqs] and num_seqs [1] are DEVICE
 *     int32 arrays, read by the planner kernel when it runs, so the caller may
 *     rewrite them (and q / k_new / v_new) between replays of a captured
 *     graph.  Entries past num_seqs are not read.
 *   dims->total_q_tokens is a capacity T: q, k_new, v_new, out (and lse)
 *     have T rows, cu_q_lens[num_seqs] <= T, and rows from cu_q_lens[num_seqs]
 *     on are not written.  page_table has max_seqs rows.
 *   No distribution: sequences are routed by q_len (1: decode kernel, > 1:
 *     prefill kernel, 0: nothing); fp32 I/O runs on the generic kernel.
 *   workspace: caller-owned device memory, 256-byte aligned, of at least
 *     rpa_device_workspace_size(dims, max_seqs) bytes (measured with the same
 *     option values), else RPA_ERR_WORKSPACE.  Calls that share a workspace
 *     must be ordered on the device.  The library allocates nothing.
 *   dev_flags: device uint32 that receives RPA_DEV_* bits (OR-ed in, never
 *     cleared), or NULL to drop them.  Lengths that rpa_forward would reject
 *     with RPA_ERR_LENGTHS set RPA_DEV_BAD_LENGTHS and the call writes
 *     nothing.
 *   The kernels launched, their grids (sized for the workspace's capacity)
 *     and arguments depend only on the pointers, dims, max_seqs, scale,
 *     causal and the option values, never on the lengths: the host neither
 *     reads device memory nor waits, so the call can be captured into a CUDA
 *     graph and replayed.  The planner kernel makes the per-batch choices
 *     rpa_forward's host planner makes (packing of short decode sequences,
 *     the producer layout of the head_dim <= 128 prefill kernel) by the same
 *     rules, from the device-resident lengths.
 * Results (out, lse, cache contents) are those rpa_forward gives for the same
 * batch.  max_seqs == 0 or T == 0 is a successful no-op.  Host-side checks
 * (scale, dims, null pointers, workspace) return RPA_ERR_* before anything is
 * queued; RPA_ERR_CUDA if a launch failed.
 */
RPA_API int rpa_forward_device(const void *q, const void *k_new,
                               const void *v_new, void *k_cache,
                               void *v_cache, const int32_t *page_table,
                               const int32_t *cu_q_lens,
                               const int32_t *kv_lens,
                               const int32_t *num_seqs, int32_t max_seqs,
                               float scale, int32_t causal, void *out,
                               float *lse, const rpa_dims *dims,
                               void *workspace, int64_t workspace_bytes,
                               uint32_t *dev_flags, void *stream);

/*
 * rpa_forward_host -- rpa_forward for a caller whose inputs and results are
 * in host memory: q, k_new, v_new, page_table, out and lse are HOST pointers
 * (same shapes and layouts as in rpa_forward); k_cache and v_cache stay
 * DEVICE buffers (the cache is resident on the GPU).  cu_q_lens, kv_lens and
 * distribution are host arrays as in rpa_forward.
 *
 * The operation is rpa_forward's (the same passages define it); the pages
 * run it on device-resident data and say nothing of host buffers.  The call
 * copies the new tokens in, runs the attention pass and copies out and lse
 * back, queued on `stream` and the library's own streams, and returns
 * without waiting: the host results are complete once `stream` has reached
 * the end of the call (e.g. after cudaStreamSynchronize(stream)).  The host
 * inputs must not be modified, nor the results read, before then.
 * Page-locked host memory (cudaMallocHost or cudaHostRegister) lets the
 * copies run asynchronously and overlap the kernels; with pageable memory
 * the results are the same, the copies do not overlap and the call may
 * return only after some of them have finished.
 *
 * Overlap: the batch is cut into at most RPA_HOST_MAX_GROUPS groups of whole
 * consecutive sequences (rpa_host_groups gives the cut; batches with under
 * 8 MiB of copies are one group, which runs entirely on `stream`).  With
 * several groups, one library copy stream takes the page table and the
 * first group's inputs, then all groups' plans, then the other groups'
 * inputs; each group's kernels start once its own inputs have arrived
 * (groups of decode sequences only on `stream`, the others on a library
 * stream of the highest priority, so they may run concurrently), and its
 * results go back on a library copy stream as soon as it is done.  The call
 * joins every library stream back into `stream` before it returns.
 *
 * Results: the cache update is bit-identical to rpa_forward's; out and lse
 * are those of rpa_forward run on each group (the same exact attention; the
 * decode split-KV work split, and therefore the fp32 rounding order, can
 * differ from one call over the whole batch).
 *
 * Workspace: per device, device staging for a call's inputs, results,
 * plans and split-KV partials, and two pinned plan buffers (all grown on
 * demand, kept until the process exits), plus rpa_forward's error word.
 * Successive calls are ordered on the device against each other even on
 * different streams.  Returns RPA_OK or an RPA_ERR_* code; all validation
 * (rpa_forward's, over the whole batch) happens before anything is queued.
 * RPA_ERR_CUDA / RPA_ERR_OOM after that point leave earlier groups' results
 * possibly written.
 */
#define RPA_HOST_MAX_GROUPS 32
RPA_API int rpa_forward_host(const void *q, const void *k_new,
                             const void *v_new, void *k_cache, void *v_cache,
                             const int32_t *page_table,
                             const int32_t *cu_q_lens, const int32_t *kv_lens,
                             int32_t num_seqs, const int32_t *distribution,
                             float scale, int32_t causal, void *out,
                             float *lse, const rpa_dims *dims, void *stream);

/*
 * rpa_host_groups -- the sequence groups rpa_forward_host would use for this
 * batch: *num_groups groups, group g holding sequences [bounds[g],
 * bounds[g+1]), bounds[0] = 0, bounds[*num_groups] = num_seqs.  bounds must
 * hold RPA_HOST_MAX_GROUPS + 1 entries.  with_lse != 0 counts lse in the
 * copy sizes (as a non-NULL lse does).  Host only; RPA_OK, or the RPA_ERR_*
 * code of bad dims or cu_q_lens (not starting at 0, decreasing, or not
 * ending at total_q_tokens).  num_seqs == 0 gives 0 groups.
 */
RPA_API int rpa_host_groups(const int32_t *cu_q_lens, int32_t num_seqs,
                            const rpa_dims *dims, int32_t with_lse,
                            int32_t *bounds, int32_t *num_groups);

#ifdef __cplusplus
}
#endif

#endif /* RPA_H */
