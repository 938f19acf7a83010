// noalloc.cu -- rpa_decode_noalloc: the decode path for callers that must
// not allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is off limits -- inside a
// custom allocator or memory pool that is itself servicing a request, in a
// process whose device memory is fully reserved up front by a serving
// framework, or under a memory budget that forbids the library from growing
// its own workspace.  rpa_forward grows a per-device workspace (plan buffers,
// split-KV partials, an error word, pinned staging) on demand; this entry
// point instead keeps all of its scratch in one fixed, file-scope device
// array that is part of the library image, and calls no cudaMalloc,
// cudaFree, cudaMallocHost or other allocating routine.
//
// Cost of that choice: the array (kScratchBytes) is reserved on every GPU
// that loads this part of the library, until the process exits, and a batch
// whose plan does not fit is rejected with RPA_ERR_SCRATCH_LIMIT.  All calls
// share the one array, so calls that can overlap on the GPU (different
// streams, or different host threads on the same device without ordering)
// race on it; callers must order them.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "host_common.h"
#include "kernels.h"
#include "plan.h"
#include "rpa.h"

namespace rpa {
namespace {

// Scratch layout (bytes): [error word | pad to 256][decode items][combine
// items][partial outputs, fp32][partial lse, fp32].
constexpr int64_t kScratchBytes = 16ll << 20;
constexpr int64_t kMaxItems = 8192;      // decode work items
// sequences needing the combine: each has at least two work items, so the
// item limit keeps them within half of it
constexpr int64_t kMaxCombine = kMaxItems / 2;
constexpr int64_t kItemsOff = 256;
constexpr int64_t kCombineOff = kItemsOff + kMaxItems * (int64_t)sizeof(DecodeItem);
constexpr int64_t kPartialOff = kCombineOff + kMaxCombine * (int64_t)sizeof(CombineItem);
constexpr int64_t kPartialFloats = (kScratchBytes - kPartialOff) / 4;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};
// Recorded after each call's plan copies; the next call waits for it before
// it refills the host staging below.  Created once per device at set-up.
cudaEvent_t g_staged[kMaxDevices] = {};
bool g_staged_pending[kMaxDevices] = {};

// Host staging for the plan (pageable, static).  The copies from it are
// asynchronous; the event above keeps a later call from rewriting it before
// the copy engine or driver has read it, whenever the driver reads it.
DecodeItem g_items[kMaxItems];
CombineItem g_combine[kMaxCombine];

}  // namespace
}  // namespace rpa

using namespace rpa;

extern "C" RPA_API int rpa_decode_noalloc(const void *q, const void *k_new, const void *v_new,
                                          void *k_cache, void *v_cache, const int32_t *page_table,
                                          const int32_t *kv_lens, int32_t num_seqs, float scale,
                                          void *out, float *lse, const rpa_dims *dims,
                                          uint32_t *dev_flags, void *stream_ptr) {
  cudaStream_t stream = (cudaStream_t)stream_ptr;
  // ---- validation (host only)
  if (dims == nullptr || num_seqs < 0) return RPA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return RPA_ERR_INVALID_ARG;
  if (dims->dtype != RPA_BF16) return RPA_ERR_UNSUPPORTED;
  if (dims->num_q_heads <= 0 || dims->num_kv_heads <= 0 || dims->num_pages <= 0 ||
      dims->max_pages_per_seq <= 0)
    return RPA_ERR_INVALID_ARG;
  const int P = dims->page_size, D = dims->head_dim;
  if (D != 64 && D != 128 && D != 256) return RPA_ERR_UNSUPPORTED;
  if (P < 8 || P > 256 || (P & (P - 1)) != 0) return RPA_ERR_UNSUPPORTED;
  if (dims->num_q_heads % dims->num_kv_heads != 0 || dims->num_q_heads / dims->num_kv_heads > 16)
    return RPA_ERR_UNSUPPORTED;
  if (dims->total_q_tokens != num_seqs) return RPA_ERR_LENGTHS;   // one new token per sequence
  if (num_seqs == 0) return RPA_OK;
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !page_table || !kv_lens || !out)
    return RPA_ERR_INVALID_ARG;
  const int64_t cap = (int64_t)dims->max_pages_per_seq * P;
  for (int32_t s = 0; s < num_seqs; ++s)
    if (kv_lens[s] < 1 || kv_lens[s] > cap) return RPA_ERR_LENGTHS;

  // ---- sizes against the fixed scratch (before touching any device)
  const int G = dims->num_q_heads / dims->num_kv_heads;
  const int64_t per_partial = (int64_t)dims->num_kv_heads * G * (D + 1);
  // 16-token blocks per work item: rpa_forward's (RPA_OPT_DECODE_CHUNK_BLOCKS)
  const int64_t chunk = decode_chunk_blocks();
  int64_t n_items = 0, n_partials = 0, n_combine = 0;
  for (int32_t s = 0; s < num_seqs; ++s) {
    const int64_t nsplit = decode_items_of(kv_lens[s], chunk);
    n_items += nsplit;
    if (nsplit > 1) {
      n_partials += nsplit;
      ++n_combine;
    }
  }
  if (n_items > kMaxItems || n_combine > kMaxCombine || n_partials * per_partial > kPartialFloats)
    return RPA_ERR_SCRATCH_LIMIT;

  // The plan goes up from host arrays that the next call rewrites, and the
  // kernels are sized for this batch: a call recorded into a CUDA graph
  // would replay whatever plan the arrays hold then.  Refuse capture.
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &capture) != cudaSuccess || capture != cudaStreamCaptureStatusNone)
    return RPA_ERR_INVALID_ARG;

  std::lock_guard<std::mutex> lock(g_mu);
  // ---- one-time set-up per device: the device address of the array and
  // the staging event
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RPA_ERR_CUDA;
  if (g_scratch_ptr[dev] == nullptr) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return RPA_ERR_CUDA;
    if (g_staged[dev] == nullptr &&
        cudaEventCreateWithFlags(&g_staged[dev], cudaEventDisableTiming) != cudaSuccess)
      return RPA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  unsigned char *scratch = static_cast<unsigned char *>(g_scratch_ptr[dev]);
  // the previous call's copies must have read the staging before it changes
  // (the arrays are shared by every device: wait for each one's last copy)
  for (int d = 0; d < kMaxDevices; ++d) {
    if (!g_staged_pending[d]) continue;
    if (cudaEventSynchronize(g_staged[d]) != cudaSuccess) return RPA_ERR_CUDA;
    g_staged_pending[d] = false;
  }

  // ---- plan: near-equal chunks of at most `chunk` 16-token blocks per
  // sequence, exactly as rpa_forward's planner cuts them
  int32_t ni = 0, nc = 0, np = 0;
  for (int32_t s = 0; s < num_seqs; ++s) {
    const int32_t made = fill_decode_items(s, s, kv_lens[s], chunk, np, g_items + ni, g_combine + nc);
    ni += made;
    if (made > 1) {
      np += made;
      ++nc;
    }
  }

  // longest items first (the kernel takes items in grid order, so the short
  // ones fill the last wave); std::sort works in place and allocates nothing
  std::sort(g_items, g_items + ni, [](const DecodeItem &x, const DecodeItem &y) {
    return x.blk_end - x.blk_begin > y.blk_end - y.blk_begin;
  });
  uint32_t *err = dev_flags ? dev_flags : reinterpret_cast<uint32_t *>(scratch);
  DecodeItem *d_items = reinterpret_cast<DecodeItem *>(scratch + kItemsOff);
  CombineItem *d_combine = reinterpret_cast<CombineItem *>(scratch + kCombineOff);
  float *part_o = reinterpret_cast<float *>(scratch + kPartialOff);
  float *part_lse = part_o + (int64_t)np * dims->num_kv_heads * G * D;
  // The scratch error word keeps the previous call's bits: clear it.
  if (dev_flags == nullptr && cudaMemsetAsync(err, 0, sizeof(uint32_t), stream) != cudaSuccess)
    return RPA_ERR_CUDA;
  if (cudaMemcpyAsync(d_items, g_items, (size_t)ni * sizeof(DecodeItem), cudaMemcpyHostToDevice, stream) !=
      cudaSuccess)
    return RPA_ERR_CUDA;
  if (nc > 0 && cudaMemcpyAsync(d_combine, g_combine, (size_t)nc * sizeof(CombineItem),
                                cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return RPA_ERR_CUDA;
  if (cudaEventRecord(g_staged[dev], stream) != cudaSuccess) return RPA_ERR_CUDA;
  g_staged_pending[dev] = true;

  Problem pb{};
  pb.q = q;
  pb.k_new = k_new;
  pb.v_new = v_new;
  pb.k_cache = k_cache;
  pb.v_cache = v_cache;
  pb.page_table = page_table;
  pb.out = out;
  pb.lse = lse;
  pb.err = err;
  pb.hq = dims->num_q_heads;
  pb.hkv = dims->num_kv_heads;
  pb.d = D;
  pb.p = P;
  pb.num_pages = dims->num_pages;
  pb.max_pages = dims->max_pages_per_seq;
  pb.dtype = RPA_BF16;
  pb.causal = 1;
  pb.scale = scale;
  cudaError_t e = launch_decode(pb, d_items, ni, part_o, part_lse, false, stream);
  if (e == cudaSuccess && nc > 0) e = launch_combine(pb, d_combine, nc, part_o, part_lse, stream, false);
  return e == cudaSuccess ? RPA_OK : RPA_ERR_CUDA;
}
