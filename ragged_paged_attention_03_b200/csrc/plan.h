// plan.h -- work descriptors the host planner writes and the kernels read.
//
// One rpa_forward call uploads one plan blob (a single host-to-device copy);
// every kernel of the call reads its own section of it.  All records are
// plain int32 so the blob has no padding surprises between host and device.
#pragma once
#include <stdint.h>

#include "rpa.h"

namespace rpa {

constexpr int kDecodeBlock = 16;   // tokens per decode block (one MMA M-tile)

// A sequence handled by the generic (SIMT, any dtype) kernel.
struct GenericSeq {
  int32_t seq;         // row of the page table
  int32_t q_start;     // first global token row
  int32_t q_len;
  int32_t kv_len;
  int32_t row_prefix;  // first generic row of this sequence (prefix over q_len)
  int32_t pad[3];
};

// One decode work item: a chunk [blk_begin, blk_end) of 16-token blocks of
// one decode sequence, for every KV head (grid.y = Hkv).  Blocks cover the
// cached context [0, kv_len - 1); the new token (position kv_len - 1) is
// taken from k_new by the item that owns the last block, which also writes
// it into the cache.
struct DecodeItem {
  int32_t seq;        // row of the page table
  int32_t token;      // global token row of the query / new token
  int32_t kv_len;
  int32_t blk_begin;
  int32_t blk_end;    // exclusive; the last item's range includes the block
                      // that holds position kv_len - 1
  int32_t partial;    // >= 0: index of this item's partial-result slot;
                      // -1: the item covers the whole sequence
  int32_t owns_new;   // 1 if this item takes and stores the new token
  int32_t pad;
};

// One decode sequence whose chunks must be merged by the LSE combine.
struct CombineItem {
  int32_t token;          // global token row
  int32_t first_partial;  // partial slots first_partial .. + nsplit - 1
  int32_t nsplit;
  int32_t pad;
};

// One prefill tile: `rows` consecutive new tokens of one sequence, all
// query heads of one KV head group handled by grid.y.
struct PrefillTile {
  int32_t seq;        // row of the page table
  int32_t q_start;    // global token row of the sequence's first new token
  int32_t q_len;
  int32_t kv_len;
  int32_t tile_row;   // first new-token index (0-based within the sequence)
  int32_t rows;       // rows in this tile (<= tile height)
  int32_t writes;     // new-token block count this tile stores to the cache
  int32_t pad;
};

// Device-planned calls (rpa_forward_device): the planner kernel writes the
// work counts into a header of int32 slots; each kernel of the call is
// launched with a grid sized for the workspace's capacity and bounds its work
// by its slot (the persistent head_dim <= 128 prefill kernel by an empty tile,
// rows == 0, after the last one).  Host-planned calls pass no header.
enum DeviceCount {
  kCntDecode = 0,       // decode work items
  kCntPacked = 1,       // packed (four per CTA) decode items
  kCntCombine = 2,      // combine rows
  kCntPrefill = 3,      // prefill tiles
  kCntGenericSeqs = 4,  // generic-kernel sequences
  kCntGenericRows = 5,  // generic-kernel rows
  kCntPartials = 6,     // split-KV partial slots in use
  kCntPrefillSplit = 7, // 1: the head_dim <= 128 prefill kernel gives K and V
                        // a producer warp each (its split build)
  kCntSlots = 8
};

// Offsets (in int32 units) of each section inside the plan blob.
struct PlanLayout {
  int64_t generic_off, n_generic_seqs, n_generic_rows;
  int64_t decode_off, n_decode_items;
  int64_t decode_packed_off, n_decode_packed;   // short whole sequences, four per CTA
  int64_t combine_off, n_combine;
  int64_t prefill_off, n_prefill_tiles;
  int64_t n_partials;      // partial slots (per KV head) needed
  int64_t total_words;
};

}  // namespace rpa
