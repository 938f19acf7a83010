// forward_internal.h -- the two halves of rpa_forward, for entry points that
// upload their plans themselves (host_io.cu): the host planner, and the
// kernel launches of a batch whose plan is already in device memory.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "kernels.h"
#include "plan.h"
#include "rpa.h"

namespace rpa {

// The host planner's result: per-kernel work lists and their blob layout.
struct HostPlan {
  std::vector<GenericSeq> generic;
  std::vector<DecodeItem> decode;
  std::vector<DecodeItem> decode_packed;   // whole short sequences, four per CTA
  std::vector<CombineItem> combine;
  std::vector<PrefillTile> prefill;
  int32_t n_generic_rows = 0;
  int32_t n_partials = 0;
  int32_t decode_max_splits = 0;
  int32_t num_decode = 0, num_prefill = 0, num_generic = 0, num_empty = 0;
  int64_t prefill_ctx_tokens = 0, prefill_new_tokens = 0;
  PlanLayout layout{};
};

// Plans a batch whose dims, lengths and distribution have been validated.
void build_plan(const int32_t *cu, const int32_t *kv, int32_t n, const int32_t *dist,
                const rpa_dims *d, HostPlan &hp);
// Writes the plan blob (hp.layout.total_words int32 words) to dst.
void serialize(const HostPlan &hp, int32_t *dst);
// Split-KV partial floats the plan's decode items write (outputs, then lse).
int64_t plan_partial_floats(const HostPlan &hp, const rpa_dims &d);
// The kernels' view of one call (err is set by launch_planned).
Problem problem_of(const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                   const int32_t *page_table, void *out, float *lse, const rpa_dims &d, float scale,
                   int32_t causal);
// Queues the kernels of a planned batch on `stream`, exactly as rpa_forward
// does after its plan upload: dev_plan holds the blob, partials has
// plan_partial_floats(hp, dims) floats.  RPA_OK, RPA_ERR_CUDA or the code of
// a failed workspace initialisation.
int launch_planned(const HostPlan &hp, const int32_t *dev_plan, float *partials, Problem pb,
                   cudaStream_t stream);

}  // namespace rpa
