// device_plan.cu -- rpa_forward_device: the metadata pass on the GPU, so that
// a whole attention call is a fixed sequence of kernel launches that a CUDA
// graph can hold and replay while the lengths change.
//
// The pages propose moving the kernel's scalar metadata work (sequence
// bookkeeping, tile boundaries) off the main compute path, to the TPU's
// SparseCore (RPA talk summary, rocketrecap.com, 00:16:06 and the roadmap
// at 00:18:14).  On
// B200 the counterpart is a one-CTA planner kernel on the same stream: it
// reads cu_q_lens / kv_lens / num_seqs from device memory, validates them,
// routes every sequence (decode: one new token; prefill / chunked prefill:
// more) and writes the same work descriptors the host planner of
// rpa_forward builds, into a caller-owned workspace.  The attention kernels
// that follow are launched with grids sized for the workspace's capacity and
// bound their work by the counts the planner wrote, so no launch parameter
// depends on the lengths and the host never waits for the device.
//
// Work order: decode items and prefill tiles are placed longest first (a
// counting sort on the item's block count, and on the tile's visible key
// range in 128-key bins), like the host planner's sorts; items of equal key
// land in any order, which changes no result.
#include <cmath>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "host_common.h"
#include "kernels.h"
#include "plan.h"
#include "rpa.h"

namespace rpa {
namespace {

constexpr int kPlanThreads = 1024;
constexpr int kLenBins = kMaxDecodeChunkBlocks + 1;  // decode item length in blocks
constexpr int kTileBins = 1024;                      // prefill tile key range / 128
constexpr int64_t kAlign = 256;
constexpr int64_t kErrOffset = 128;                  // error word in the header

int64_t align_up(int64_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Per device: the highest-priority stream the prefill kernel runs on, next
// to the decode kernels on the caller's stream, and the fork / join events.
// Captured into a graph these become two parallel branches.
struct SideStream {
  std::mutex mu;
  bool init = false;
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxDevices = 64;
SideStream g_side[kMaxDevices];

bool side_init(SideStream &s) {
  if (s.init) return true;
  int lo = 0, hi = 0;
  if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) hi = 0;
  if (cudaStreamCreateWithPriority(&s.side, cudaStreamNonBlocking, hi) != cudaSuccess ||
      cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming) != cudaSuccess)
    return false;
  s.init = true;
  return true;
}

// Capacities and byte offsets of a device-planned call's workspace.  Every
// bound follows from the geometry alone: a decode sequence takes one new
// token and at most max_split chunks; a prefill sequence takes at least two
// new tokens and ceil(q_len / item_rows) tiles.
struct DeviceLayout {
  int64_t cap_items = 0, cap_packed = 0, cap_combine = 0, cap_tiles = 0, cap_partials = 0, cap_generic = 0;
  int64_t items = 0, packed = 0, combine = 0, tiles = 0, generic = 0, part_o = 0, part_lse = 0;
  int64_t total = 0;
  int32_t chunk = 0, pack = 0;
};

DeviceLayout device_layout(const rpa_dims *d, int32_t max_seqs) {
  DeviceLayout L;
  L.chunk = (int32_t)decode_chunk_blocks();
  L.pack = (int32_t)decode_pack_blocks();
  const int64_t T = d->total_q_tokens;
  const int G = d->num_q_heads / d->num_kv_heads;
  if (d->dtype == RPA_BF16) {
    const int64_t n_dec = std::min<int64_t>(max_seqs, T);
    const int64_t max_blk = ((int64_t)d->max_pages_per_seq * d->page_size + 15) / 16;
    const int64_t max_split = (max_blk + L.chunk - 1) / L.chunk;
    const int64_t rows = prefill_item_rows(d->head_dim);
    L.cap_items = n_dec * max_split;
    L.cap_packed = L.pack > 0 ? n_dec : 0;
    L.cap_combine = max_split > 1 ? n_dec : 0;
    L.cap_partials = max_split > 1 ? n_dec * max_split : 0;
    L.cap_tiles = T >= 2 && max_seqs > 0 ? (T + rows - 1) / rows + std::min<int64_t>(max_seqs, T / 2) : 0;
  } else {
    L.cap_generic = max_seqs;
  }
  int64_t off = kAlign;  // header: kCntSlots counts, the error word at kErrOffset
  L.items = off;
  off = align_up(off + L.cap_items * (int64_t)sizeof(DecodeItem));
  L.packed = off;
  off = align_up(off + L.cap_packed * (int64_t)sizeof(DecodeItem));
  L.combine = off;
  off = align_up(off + L.cap_combine * (int64_t)sizeof(CombineItem));
  L.tiles = off;
  off = align_up(off + L.cap_tiles * (int64_t)sizeof(PrefillTile));
  L.generic = off;
  off = align_up(off + L.cap_generic * (int64_t)sizeof(GenericSeq));
  L.part_o = off;
  off = align_up(off + L.cap_partials * d->num_kv_heads * G * (int64_t)d->head_dim * 4);
  L.part_lse = off;
  off = align_up(off + L.cap_partials * d->num_kv_heads * G * 4);
  L.total = off;
  return L;
}

struct PlanArgs {
  const int32_t *cu, *kv, *num_seqs;
  int32_t max_seqs, T, P, max_pages, hkv, chunk, pack, item_rows, bf16, loaders;
  int32_t *counts;
  uint32_t *err;
  DecodeItem *items, *packed;
  CombineItem *combine;
  PrefillTile *tiles;
  GenericSeq *generic;
  int64_t cap_items, cap_packed, cap_tiles;
};

// One warp turns a histogram into start offsets in place, largest key first
// (bin b starts after every entry of bins above b); returns the total.
__device__ int offsets_largest_first(int *h, int nb, int lane) {
  const int per = (nb + 31) / 32;
  const int i0 = lane * per, i1 = min(nb, i0 + per);   // positions in descending key order
  int sum = 0;
  for (int i = i0; i < i1; ++i) sum += h[nb - 1 - i];
  int incl = sum;
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int run = incl - sum;
  for (int i = i0; i < i1; ++i) {
    const int b = nb - 1 - i;
    const int c = h[b];
    h[b] = run;
    run += c;
  }
  return __shfl_sync(0xffffffffu, incl, 31);
}

__device__ __forceinline__ void write_counts(int32_t *counts, int dec, int packed, int comb, int tiles,
                                             int gseqs, int grows, int partials, int split) {
  counts[kCntDecode] = dec;
  counts[kCntPacked] = packed;
  counts[kCntCombine] = comb;
  counts[kCntPrefill] = tiles;
  counts[kCntGenericSeqs] = gseqs;
  counts[kCntGenericRows] = grows;
  counts[kCntPartials] = partials;
  counts[kCntPrefillSplit] = split;
}

__global__ void __launch_bounds__(kPlanThreads) device_plan_kernel(const PlanArgs a) {
  __shared__ int h_items[kLenBins], h_packed[kLenBins], h_tiles[kTileBins];
  __shared__ int s_short, s_partials, s_combine, s_total[3];
  __shared__ unsigned long long s_ctx, s_new;   // prefill rows: cached context, new tokens
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kLenBins; i += kPlanThreads) h_items[i] = h_packed[i] = 0;
  for (int i = tid; i < kTileBins; i += kPlanThreads) h_tiles[i] = 0;
  if (tid == 0) {
    s_short = s_partials = s_combine = 0;
    s_ctx = s_new = 0;
  }

  // ---- validation (the host path's rules) and the count of packable sequences
  int n = *a.num_seqs;
  int bad = n < 0 || n > a.max_seqs;
  if (bad) n = 0;
  if (tid == 0 && (a.cu[0] != 0 || a.cu[n] > a.T)) bad = 1;
  const int64_t cap = (int64_t)a.max_pages * a.P;
  int my_short = 0;
  for (int s = tid; s < n; s += kPlanThreads) {
    const int64_t ql = (int64_t)a.cu[s + 1] - a.cu[s], kvl = a.kv[s];
    if (ql < 0 || kvl < ql || kvl > cap) {
      bad = 1;
    } else if (a.bf16 && ql == 1) {
      const int64_t nb = (kvl + 15) >> 4;
      if (nb <= a.pack && nb <= a.chunk) ++my_short;
    }
  }
  __syncthreads();
  if (my_short) atomicAdd(&s_short, my_short);
  if (__syncthreads_or(bad)) {
    if (tid == 0) {
      write_counts(a.counts, 0, 0, 0, 0, 0, 0, 0, 0);
      atomicOr(a.err, RPA_DEV_BAD_LENGTHS);
    }
    return;
  }

  if (!a.bf16) {
    // fp32 I/O: every sequence on the generic kernel, rows in token order
    for (int s = tid; s < n; s += kPlanThreads) {
      GenericSeq g{};
      g.seq = s;
      g.q_start = a.cu[s];
      g.q_len = a.cu[s + 1] - a.cu[s];
      g.kv_len = a.kv[s];
      g.row_prefix = a.cu[s];
      a.generic[s] = g;
    }
    if (tid == 0) write_counts(a.counts, 0, 0, 0, 0, n, a.cu[n], 0, 0);
    return;
  }

  const bool packing = a.pack > 0 && (int64_t)((s_short + 3) / 4) * a.hkv >= kMinPackedCtas;
  const int R = a.item_rows;
  // ---- histograms of the sort keys
  unsigned long long my_ctx = 0, my_new = 0;
  for (int s = tid; s < n; s += kPlanThreads) {
    const int ql = a.cu[s + 1] - a.cu[s], kvl = a.kv[s];
    if (ql == 1) {
      const int nb = (kvl + 15) >> 4;
      if (packing && nb <= a.pack && nb <= a.chunk) {
        atomicAdd(&h_packed[nb], 1);
      } else {
        const int ns = (nb + a.chunk - 1) / a.chunk, per = (nb + ns - 1) / ns;
        if (ns > 1) atomicAdd(&h_items[per], ns - 1);
        atomicAdd(&h_items[nb - (ns - 1) * per], 1);
      }
    } else if (ql > 1) {
      my_ctx += (unsigned long long)(kvl - ql);
      my_new += (unsigned long long)ql;
      for (int r = 0; r < ql; r += R) {
        const int w = kvl - ql + r + min(R, ql - r);   // keys visible to the tile's last row
        atomicAdd(&h_tiles[min(w >> 7, kTileBins - 1)], 1);
      }
    }
  }
  if (my_new) {
    atomicAdd(&s_ctx, my_ctx);
    atomicAdd(&s_new, my_new);
  }
  __syncthreads();
  if (warp == 0) {
    const int t = offsets_largest_first(h_items, kLenBins, lane);
    if (lane == 0) s_total[0] = t;
  } else if (warp == 1) {
    const int t = offsets_largest_first(h_packed, kLenBins, lane);
    if (lane == 0) s_total[1] = t;
  } else if (warp == 2) {
    const int t = offsets_largest_first(h_tiles, kTileBins, lane);
    if (lane == 0) s_total[2] = t;
  }
  __syncthreads();
  // the capacities bound these by construction; a mismatch writes nothing
  if (s_total[0] > a.cap_items || s_total[1] > a.cap_packed || s_total[2] > a.cap_tiles) {
    if (tid == 0) {
      write_counts(a.counts, 0, 0, 0, 0, 0, 0, 0, 0);
      atomicOr(a.err, RPA_DEV_BAD_LENGTHS);
    }
    return;
  }

  // ---- descriptors, each at its key's next free place
  for (int s = tid; s < n; s += kPlanThreads) {
    const int q0 = a.cu[s], ql = a.cu[s + 1] - q0, kvl = a.kv[s];
    if (ql == 1) {
      const int nb = (kvl + 15) >> 4;
      DecodeItem it{};
      it.seq = s;
      it.token = q0;
      it.kv_len = kvl;
      if (packing && nb <= a.pack && nb <= a.chunk) {
        it.blk_begin = 0;
        it.blk_end = nb;
        it.partial = -1;
        it.owns_new = 1;
        a.packed[atomicAdd(&h_packed[nb], 1)] = it;
        continue;
      }
      const int ns = (nb + a.chunk - 1) / a.chunk, per = (nb + ns - 1) / ns;
      int first = -1;
      if (ns > 1) {
        first = atomicAdd(&s_partials, ns);
        CombineItem c{};
        c.token = q0;
        c.first_partial = first;
        c.nsplit = ns;
        a.combine[atomicAdd(&s_combine, 1)] = c;
      }
      for (int k = 0; k < ns; ++k) {
        it.blk_begin = k * per;
        it.blk_end = min(nb, it.blk_begin + per);
        it.partial = ns > 1 ? first + k : -1;
        it.owns_new = it.blk_end == nb ? 1 : 0;
        a.items[atomicAdd(&h_items[it.blk_end - it.blk_begin], 1)] = it;
      }
    } else if (ql > 1) {
      for (int r = 0; r < ql; r += R) {
        PrefillTile t{};
        t.seq = s;
        t.q_start = q0;
        t.q_len = ql;
        t.kv_len = kvl;
        t.tile_row = r;
        t.rows = min(R, ql - r);
        const int w = kvl - ql + r + t.rows;
        a.tiles[atomicAdd(&h_tiles[min(w >> 7, kTileBins - 1)], 1)] = t;
      }
    }
  }
  // empty tiles after the last one end the persistent prefill kernel's list
  for (int64_t i = s_total[2] + tid; i < a.cap_tiles; i += kPlanThreads) a.tiles[i] = PrefillTile{};
  __syncthreads();
  // producer layout of the head_dim <= 128 prefill kernel, the host planner's
  // rule: one warp per operand when the prefill rows are mostly cached context
  const int split = a.loaders == 2 || (a.loaders != 1 && s_ctx > s_new);
  if (tid == 0) write_counts(a.counts, s_total[0], s_total[1], s_combine, s_total[2], 0, 0, s_partials, split);
}

}  // namespace
}  // namespace rpa

using namespace rpa;

extern "C" RPA_API int rpa_device_workspace_size(const rpa_dims *dims, int32_t max_seqs, int64_t *bytes) {
  if (bytes == nullptr) return RPA_ERR_INVALID_ARG;
  *bytes = 0;
  const int rc = validate_dims(dims);
  if (rc) return rc;
  if (max_seqs < 0) return RPA_ERR_INVALID_ARG;
  *bytes = device_layout(dims, max_seqs).total;
  return RPA_OK;
}

extern "C" RPA_API int rpa_forward_device(const void *q, const void *k_new, const void *v_new, void *k_cache,
                                          void *v_cache, const int32_t *page_table, const int32_t *cu_q_lens,
                                          const int32_t *kv_lens, const int32_t *num_seqs, int32_t max_seqs,
                                          float scale, int32_t causal, void *out, float *lse,
                                          const rpa_dims *dims, void *workspace, int64_t workspace_bytes,
                                          uint32_t *dev_flags, void *stream_ptr) {
  cudaStream_t stream = (cudaStream_t)stream_ptr;
  if (!(scale > 0.f) || !std::isfinite(scale)) return RPA_ERR_INVALID_ARG;
  int rc = validate_dims(dims);
  if (rc) return rc;
  if (max_seqs < 0) return RPA_ERR_INVALID_ARG;
  if (max_seqs == 0 || dims->total_q_tokens == 0) return RPA_OK;  // no sequence can hold a new token
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !page_table || !cu_q_lens || !kv_lens || !num_seqs ||
      !out || !workspace)
    return RPA_ERR_INVALID_ARG;
  const DeviceLayout L = device_layout(dims, max_seqs);
  // launch geometry: item counts in int, prefill_kernel tiles on grid.y
  if (L.cap_items > INT32_MAX / 8 || L.cap_tiles > 65535 || (int64_t)max_seqs * dims->num_q_heads > INT32_MAX / 32)
    return RPA_ERR_UNSUPPORTED;
  if (workspace_bytes < L.total || reinterpret_cast<uintptr_t>(workspace) % kAlign != 0) return RPA_ERR_WORKSPACE;

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int32_t *counts = reinterpret_cast<int32_t *>(ws);
  PlanArgs a{};
  a.cu = cu_q_lens;
  a.kv = kv_lens;
  a.num_seqs = num_seqs;
  a.max_seqs = max_seqs;
  a.T = dims->total_q_tokens;
  a.P = dims->page_size;
  a.max_pages = dims->max_pages_per_seq;
  a.hkv = dims->num_kv_heads;
  a.chunk = L.chunk;
  a.pack = L.pack;
  a.item_rows = prefill_item_rows(dims->head_dim);
  a.bf16 = dims->dtype == RPA_BF16 ? 1 : 0;
  a.loaders = (int32_t)prefill_loaders();
  a.counts = counts;
  a.err = dev_flags ? dev_flags : reinterpret_cast<uint32_t *>(ws + kErrOffset);
  a.items = reinterpret_cast<DecodeItem *>(ws + L.items);
  a.packed = reinterpret_cast<DecodeItem *>(ws + L.packed);
  a.combine = reinterpret_cast<CombineItem *>(ws + L.combine);
  a.tiles = reinterpret_cast<PrefillTile *>(ws + L.tiles);
  a.generic = reinterpret_cast<GenericSeq *>(ws + L.generic);
  a.cap_items = L.cap_items;
  a.cap_packed = L.cap_packed;
  a.cap_tiles = L.cap_tiles;

  Problem pb{};
  pb.q = q;
  pb.k_new = k_new;
  pb.v_new = v_new;
  pb.k_cache = k_cache;
  pb.v_cache = v_cache;
  pb.page_table = page_table;
  pb.out = out;
  pb.lse = lse;
  pb.err = a.err;
  pb.hq = dims->num_q_heads;
  pb.hkv = dims->num_kv_heads;
  pb.d = dims->head_dim;
  pb.p = dims->page_size;
  pb.num_pages = dims->num_pages;
  pb.max_pages = dims->max_pages_per_seq;
  pb.dtype = dims->dtype;
  pb.causal = causal ? 1 : 0;
  pb.scale = scale;
  pb.total_q = dims->total_q_tokens;
  pb.dev_counts = counts;

  device_plan_kernel<<<1, kPlanThreads, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  float *part_o = reinterpret_cast<float *>(ws + L.part_o);
  float *part_lse = reinterpret_cast<float *>(ws + L.part_lse);
  if (dims->dtype == RPA_BF16) {
    // prefill and decode concurrently, as rpa_forward runs a mixed batch:
    // prefill on the highest-priority side stream (its CTAs are placed
    // first), decode on the caller's stream filling the SMs prefill leaves
    const bool both = L.cap_tiles > 0 && L.cap_items > 0 && concurrent_mixed();
    SideStream *ss = nullptr;
    std::unique_lock<std::mutex> lock;
    cudaStream_t pstream = stream;
    if (e == cudaSuccess && both) {
      int dev = 0;
      if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RPA_ERR_CUDA;
      ss = &g_side[dev];
      lock = std::unique_lock<std::mutex>(ss->mu);
      if (!side_init(*ss)) return RPA_ERR_CUDA;
      if (cudaEventRecord(ss->fork, stream) != cudaSuccess || cudaStreamWaitEvent(ss->side, ss->fork, 0) != cudaSuccess)
        return RPA_ERR_CUDA;
      pstream = ss->side;
    }
    if (e == cudaSuccess && L.cap_tiles > 0)
      e = launch_prefill_any(pb, a.tiles, (int)L.cap_tiles, (int)std::max<int64_t>(0, prefill_sms()), false, pstream);
    const cudaError_t ej = ss ? cudaEventRecord(ss->join, pstream) : cudaSuccess;
    if (e == cudaSuccess) e = ej;
    if (e == cudaSuccess && L.cap_items > 0)
      e = launch_decode(pb, a.items, (int)L.cap_items, part_o, part_lse, false, stream);
    if (e == cudaSuccess && L.cap_packed > 0)
      e = launch_decode(pb, a.packed, (int)L.cap_packed, part_o, part_lse, true, stream);
    if (e == cudaSuccess && L.cap_combine > 0)
      e = launch_combine(pb, a.combine, (int)L.cap_combine, part_o, part_lse, stream, false);
    // join (also after an error, so that nothing of the call runs unordered)
    if (ss && ej == cudaSuccess && cudaStreamWaitEvent(stream, ss->join, 0) != cudaSuccess && e == cudaSuccess)
      e = cudaErrorUnknown;
  } else if (e == cudaSuccess) {
    e = launch_generic(pb, a.generic, max_seqs, dims->total_q_tokens, stream);
  }
  return e == cudaSuccess ? RPA_OK : RPA_ERR_CUDA;
}
