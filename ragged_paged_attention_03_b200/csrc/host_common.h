// host_common.h -- host-side helpers shared by the entry points of the
// library (rpa_api.cu, device_plan.cu, host_io.cu): validation and the
// effective values of the process-wide planner options.
#pragma once
#include <stdint.h>

#include "kernels.h"
#include "plan.h"
#include "rpa.h"

namespace rpa {

// RPA_OK, or the RPA_ERR_* code rpa_forward returns for these dims.
int validate_dims(const rpa_dims *d);
// ... for these host lengths (cu_q_lens [n+1], kv_lens [n]) under dims d.
int validate_lengths(const int32_t *cu, const int32_t *kv, int32_t n, const rpa_dims *d);
// ... for this distribution (NULL is always valid) of valid lengths.
int validate_distribution(const int32_t *dist, const int32_t *cu, const int32_t *kv, int32_t n);

// Effective planner options (defaults and clamps applied).
int64_t decode_chunk_blocks();   // 16-token blocks per decode work item
int64_t decode_pack_blocks();    // longest packed decode sequence, 0 = never
int64_t prefill_loaders();       // RPA_OPT_PREFILL_LOADERS as set (0, 1, 2)
bool concurrent_mixed();         // RPA_OPT_CONCURRENT_MIXED >= 0
int64_t prefill_sms();           // RPA_OPT_PREFILL_SMS (<= 0: one CTA per SM)
int64_t prefill_kernel();        // RPA_OPT_PREFILL_KERNEL as set (0 .. 3)

// The prefill kernel for this head dim (RPA_OPT_PREFILL_KERNEL picks among
// the head_dim 128 ones): the same launch contract as launch_prefill2.
cudaError_t launch_prefill_any(const Problem &pb, const PrefillTile *tiles, int n_tiles, int max_ctas, bool split,
                               cudaStream_t stream);

// Decode work items of one sequence with kv_len tokens (one new token at
// global row `token`): near-equal chunks of at most `chunk` 16-token blocks,
// decode_items_of(kv_len, chunk) of them.  fill_decode_items writes them to
// items[0 .. count): the last one owns the new token; when there is more than
// one, they take partial slots first_partial .. + count - 1 and *combine (if
// not NULL) receives the combine row that merges them.  Both host planners
// (rpa_forward's and the allocation-free decode entry point's) call these.
int32_t decode_items_of(int32_t kv_len, int64_t chunk);
int32_t fill_decode_items(int32_t seq, int32_t token, int32_t kv_len, int64_t chunk, int32_t first_partial,
                          DecodeItem *items, CombineItem *combine);

// Packed decode CTAs a batch must fill before packing is used (two per SM
// of a 148-SM B200): a packed launch follows the main decode launch, so a
// few short sequences are better placed in that launch's last wave.
constexpr int kMinPackedCtas = 296;

// Largest decode work item, in 16-token blocks: 256 blocks of 16 tokens
// touch at most 4096 / 8 + 1 pages, within the decode kernel's 1024-entry
// page list.
constexpr int kMaxDecodeChunkBlocks = 256;

}  // namespace rpa
