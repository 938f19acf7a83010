// rpa_api.cu -- the C ABI of include/rpa.h: validation, the host planner,
// the per-device workspace and the kernel launches of one rpa_forward call.
//
// The planner is the B200 counterpart of the distribution-aware
// specialisation in "Ragged Paged Attention" (arXiv 2604.15464), abstract,
// technique 3: each sequence is routed to the kernel specialised for its
// shape (decode: one new token; prefill / chunked prefill: many), and the
// per-kernel work lists are built on the host, uploaded with one copy and
// consumed by the kernels.
#include <cmath>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <new>
#include <vector>

#include "host_common.h"
#include "kernels.h"
#include "forward_internal.h"
#include "plan.h"
#include "rpa.h"

namespace rpa {
namespace {

std::atomic<int64_t> g_opt_decode_chunk{0};
std::atomic<int64_t> g_opt_force_generic{0};
std::atomic<int64_t> g_opt_disable_prefill_tc{0};
std::atomic<int64_t> g_opt_prefill_sms{0};
std::atomic<int64_t> g_opt_concurrent_mixed{0};
std::atomic<int64_t> g_opt_prefill_loaders{0};
std::atomic<int64_t> g_opt_decode_pack{0};
std::atomic<int64_t> g_opt_prefill_kernel{0};

constexpr int kDefaultDecodeChunkBlocks = 192;
// Decode sequences this short (16-token blocks) run four per CTA, one per
// warp; at most kMaxPackBlocks so that a warp's page-table slice (a quarter
// of the kernel's 1024 slots) holds them at page size 8.
constexpr int kDefaultDecodePackBlocks = 64;
constexpr int kMaxPackBlocks = 120;
constexpr bool kHaveDecodeKernel = true;
constexpr bool kHavePrefillKernel = true;

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

}  // namespace

int64_t decode_chunk_blocks() {
  int64_t chunk = g_opt_decode_chunk.load();
  if (chunk <= 0) chunk = kDefaultDecodeChunkBlocks;
  return std::min<int64_t>(chunk, kMaxDecodeChunkBlocks);
}

int64_t decode_pack_blocks() {
  const int64_t pack = g_opt_decode_pack.load();
  return pack == 0 ? kDefaultDecodePackBlocks : std::min<int64_t>(std::max<int64_t>(pack, 0), kMaxPackBlocks);
}

int64_t prefill_loaders() { return g_opt_prefill_loaders.load(); }

bool concurrent_mixed() { return g_opt_concurrent_mixed.load() >= 0; }

int64_t prefill_sms() { return g_opt_prefill_sms.load(); }

int64_t prefill_kernel() { return g_opt_prefill_kernel.load(); }

int prefill_item_rows(int head_dim) {
  if (head_dim <= 128) return 256;
  return prefill_kernel() == 1 ? 128 : 256;
}

cudaError_t launch_prefill_any(const Problem &pb, const PrefillTile *tiles, int n_tiles, int max_ctas, bool split,
                               cudaStream_t stream) {
  const int64_t k = prefill_kernel();
  // head_dim 256: CTA pairs unless the one-tile kernel is asked for (its
  // items are 128 rows; prefill_item_rows follows the same choice)
  if (pb.d == 256) return k == 1 ? launch_prefill(pb, tiles, n_tiles, stream)
                                 : launch_prefill3(pb, tiles, n_tiles, max_ctas, true, stream);
  if (pb.d == 128 && (k == 2 || k == 3)) return launch_prefill3(pb, tiles, n_tiles, max_ctas, k == 2, stream);
  return launch_prefill2(pb, tiles, n_tiles, max_ctas, split, stream);
}

int32_t decode_items_of(int32_t kv_len, int64_t chunk) {
  const int64_t nblk = ((int64_t)kv_len + kDecodeBlock - 1) / kDecodeBlock;
  return (int32_t)((nblk + chunk - 1) / chunk);
}

int32_t fill_decode_items(int32_t seq, int32_t token, int32_t kv_len, int64_t chunk, int32_t first_partial,
                          DecodeItem *items, CombineItem *combine) {
  const int32_t nblk = (kv_len + kDecodeBlock - 1) / kDecodeBlock;
  const int32_t nsplit = decode_items_of(kv_len, chunk);
  const int32_t per = (nblk + nsplit - 1) / nsplit;   // ceil(nblk / per) == nsplit
  for (int32_t k = 0; k < nsplit; ++k) {
    DecodeItem &it = items[k];
    memset(&it, 0, sizeof it);
    it.seq = seq;
    it.token = token;
    it.kv_len = kv_len;
    it.blk_begin = k * per;
    it.blk_end = std::min(nblk, it.blk_begin + per);
    it.owns_new = it.blk_end == nblk ? 1 : 0;
    it.partial = nsplit > 1 ? first_partial + k : -1;
  }
  if (nsplit > 1 && combine != nullptr) {
    memset(combine, 0, sizeof *combine);
    combine->token = token;
    combine->first_partial = first_partial;
    combine->nsplit = nsplit;
  }
  return nsplit;
}

int validate_dims(const rpa_dims *d) {
  if (d == nullptr) return RPA_ERR_INVALID_ARG;
  if (d->num_q_heads <= 0 || d->num_kv_heads <= 0 || d->num_pages <= 0 ||
      d->max_pages_per_seq <= 0 || d->total_q_tokens < 0 ||
      (d->dtype != RPA_F32 && d->dtype != RPA_BF16))
    return RPA_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128 && d->head_dim != 256) return RPA_ERR_UNSUPPORTED;
  if (!is_pow2(d->page_size) || d->page_size < 8 || d->page_size > 256) return RPA_ERR_UNSUPPORTED;
  if (d->num_q_heads % d->num_kv_heads != 0) return RPA_ERR_UNSUPPORTED;
  if (d->num_q_heads / d->num_kv_heads > 16) return RPA_ERR_UNSUPPORTED;
  return RPA_OK;
}

int validate_lengths(const int32_t *cu, const int32_t *kv, int32_t n, const rpa_dims *d) {
  if (n < 0) return RPA_ERR_INVALID_ARG;
  if (n == 0) return d->total_q_tokens == 0 ? RPA_OK : RPA_ERR_LENGTHS;
  if (cu == nullptr || kv == nullptr) return RPA_ERR_INVALID_ARG;
  if (cu[0] != 0) return RPA_ERR_LENGTHS;
  const int64_t cap = (int64_t)d->max_pages_per_seq * d->page_size;
  for (int32_t s = 0; s < n; ++s) {
    int64_t ql = (int64_t)cu[s + 1] - cu[s];
    if (ql < 0 || kv[s] < ql || (int64_t)kv[s] > cap) return RPA_ERR_LENGTHS;
  }
  if (cu[n] != d->total_q_tokens) return RPA_ERR_LENGTHS;
  return RPA_OK;
}

int validate_distribution(const int32_t *dist, const int32_t *cu, const int32_t *kv, int32_t n) {
  if (dist == nullptr) return RPA_OK;
  const int32_t dd = dist[0], pp = dist[1], ss = dist[2];
  if (dd < 0 || dd > pp || pp > ss || ss != n) return RPA_ERR_DISTRIBUTION;
  for (int32_t s = 0; s < n; ++s) {
    int32_t ql = cu[s + 1] - cu[s];
    if (s < dd && ql > 1) return RPA_ERR_DISTRIBUTION;
    if (s >= dd && s < pp && ql != kv[s]) return RPA_ERR_DISTRIBUTION;
  }
  return RPA_OK;
}

namespace {

enum Route { kEmpty, kGeneric, kDecode, kPrefill };

// Kernel choice for one sequence.  With a distribution the ranges decide the
// specialisation directly; without one the lengths do.  Both give the same
// answer for consistent input, and neither affects the result.
Route route_of(int32_t ql, int32_t kvl, int dtype, int cls) {
  (void)kvl;
  if (ql == 0) return kEmpty;
  if (dtype != RPA_BF16 || g_opt_force_generic.load()) return kGeneric;
  const bool decode = cls >= 0 ? (cls == 0 || ql == 1) : ql == 1;
  if (decode) return kHaveDecodeKernel ? kDecode : kGeneric;
  if (!kHavePrefillKernel || g_opt_disable_prefill_tc.load()) return kGeneric;
  return kPrefill;
}

}  // namespace

void build_plan(const int32_t *cu, const int32_t *kv, int32_t n, const int32_t *dist,
                const rpa_dims *d, HostPlan &hp) {
  const int64_t chunk = decode_chunk_blocks();
  const int64_t pack = decode_pack_blocks();
  for (int32_t s = 0; s < n; ++s) {
    const int32_t ql = cu[s + 1] - cu[s];
    const int32_t kvl = kv[s];
    int cls = -1;
    if (dist) cls = s < dist[0] ? 0 : (s < dist[1] ? 1 : 2);
    switch (route_of(ql, kvl, d->dtype, cls)) {
      case kEmpty:
        ++hp.num_empty;
        break;
      case kGeneric: {
        GenericSeq g{};
        g.seq = s;
        g.q_start = cu[s];
        g.q_len = ql;
        g.kv_len = kvl;
        g.row_prefix = hp.n_generic_rows;
        hp.n_generic_rows += ql;
        hp.generic.push_back(g);
        ++hp.num_generic;
        break;
      }
      case kDecode: {
        ++hp.num_decode;
        const int32_t nblk = (kvl + kDecodeBlock - 1) / kDecodeBlock;
        if (nblk <= pack && nblk <= chunk) {
          // short: the whole sequence as one item of a packed CTA
          DecodeItem it{};
          it.seq = s;
          it.token = cu[s];
          it.kv_len = kvl;
          it.blk_begin = 0;
          it.blk_end = nblk;
          it.owns_new = 1;
          it.partial = -1;
          hp.decode_packed.push_back(it);
          hp.decode_max_splits = std::max(hp.decode_max_splits, 1);
          break;
        }
        const int32_t nsplit = decode_items_of(kvl, chunk);
        hp.decode_max_splits = std::max(hp.decode_max_splits, nsplit);
        const size_t at = hp.decode.size();
        hp.decode.resize(at + (size_t)nsplit);
        CombineItem c{};
        fill_decode_items(s, cu[s], kvl, chunk, hp.n_partials, hp.decode.data() + at, &c);
        if (nsplit > 1) {
          hp.n_partials += nsplit;
          hp.combine.push_back(c);
        }
        break;
      }
      case kPrefill: {
        ++hp.num_prefill;
        hp.prefill_ctx_tokens += (int64_t)kvl - ql;
        hp.prefill_new_tokens += ql;
        const int32_t item_rows = prefill_item_rows(d->head_dim);
        for (int32_t r = 0; r < ql; r += item_rows) {
          PrefillTile t{};
          t.seq = s;
          t.q_start = cu[s];
          t.q_len = ql;
          t.kv_len = kvl;
          t.tile_row = r;
          t.rows = std::min(item_rows, ql - r);
          hp.prefill.push_back(t);
        }
        break;
      }
    }
  }
  // Longest decode work items first: the kernel takes items in grid order,
  // so the short ones fill the last wave instead of trailing it (and packed
  // CTAs get four items of similar length).
  auto longer = [](const DecodeItem &a, const DecodeItem &b) {
    return a.blk_end - a.blk_begin > b.blk_end - b.blk_begin;
  };
  if ((int64_t)(hp.decode_packed.size() + 3) / 4 * d->num_kv_heads < kMinPackedCtas) {
    hp.decode.insert(hp.decode.end(), hp.decode_packed.begin(), hp.decode_packed.end());
    hp.decode_packed.clear();
  }
  std::stable_sort(hp.decode.begin(), hp.decode.end(), longer);
  std::stable_sort(hp.decode_packed.begin(), hp.decode_packed.end(), longer);
  // Heaviest prefill tiles first: with a causal mask a tile's key range ends
  // at its last row, so later tiles of a sequence carry more work.
  std::stable_sort(hp.prefill.begin(), hp.prefill.end(),
                   [](const PrefillTile &a, const PrefillTile &b) {
                     int64_t wa = (int64_t)(a.kv_len - a.q_len + a.tile_row + a.rows);
                     int64_t wb = (int64_t)(b.kv_len - b.q_len + b.tile_row + b.rows);
                     return wa > wb;
                   });
  PlanLayout &L = hp.layout;
  int64_t off = 0;
  L.generic_off = off;
  L.n_generic_seqs = (int64_t)hp.generic.size();
  L.n_generic_rows = hp.n_generic_rows;
  off += L.n_generic_seqs * (int64_t)(sizeof(GenericSeq) / 4);
  L.decode_off = off;
  L.n_decode_items = (int64_t)hp.decode.size();
  off += L.n_decode_items * (int64_t)(sizeof(DecodeItem) / 4);
  L.decode_packed_off = off;
  L.n_decode_packed = (int64_t)hp.decode_packed.size();
  off += L.n_decode_packed * (int64_t)(sizeof(DecodeItem) / 4);
  L.combine_off = off;
  L.n_combine = (int64_t)hp.combine.size();
  off += L.n_combine * (int64_t)(sizeof(CombineItem) / 4);
  L.prefill_off = off;
  L.n_prefill_tiles = (int64_t)hp.prefill.size();
  off += L.n_prefill_tiles * (int64_t)(sizeof(PrefillTile) / 4);
  L.n_partials = hp.n_partials;
  L.total_words = off;
}

void serialize(const HostPlan &hp, int32_t *dst) {
  const PlanLayout &L = hp.layout;
  if (!hp.generic.empty())
    memcpy(dst + L.generic_off, hp.generic.data(), hp.generic.size() * sizeof(GenericSeq));
  if (!hp.decode.empty())
    memcpy(dst + L.decode_off, hp.decode.data(), hp.decode.size() * sizeof(DecodeItem));
  if (!hp.decode_packed.empty())
    memcpy(dst + L.decode_packed_off, hp.decode_packed.data(), hp.decode_packed.size() * sizeof(DecodeItem));
  if (!hp.combine.empty())
    memcpy(dst + L.combine_off, hp.combine.data(), hp.combine.size() * sizeof(CombineItem));
  if (!hp.prefill.empty())
    memcpy(dst + L.prefill_off, hp.prefill.data(), hp.prefill.size() * sizeof(PrefillTile));
}

namespace {

// ---------------------------------------------------------------- workspace
//
// Per device: a ring of slots, each with a pinned host staging buffer, a
// device plan buffer, a split-KV partial buffer and an event recorded after
// the slot's last kernel.  A slot is reused only once its event has fired,
// so calls on different streams never overwrite a plan or partials that a
// queued kernel still reads.
constexpr int kSlots = 4;
constexpr int kMaxDevices = 64;

struct Slot {
  int32_t *host = nullptr;
  int32_t *dev = nullptr;
  int64_t words = 0;
  float *partial = nullptr;  // o then lse
  int64_t partial_floats = 0;
  cudaEvent_t done = nullptr;
  cudaEvent_t fork = nullptr;   // caller's stream -> side stream
  cudaEvent_t join = nullptr;   // side stream -> caller's stream
  bool pending = false;
};

struct DeviceWs {
  std::mutex mu;
  bool init = false;
  uint32_t *err = nullptr;
  cudaStream_t side = nullptr;  // prefill of mixed batches runs here
  cudaEvent_t fork = nullptr, join = nullptr;   // side-stream order for launch_planned
  int sms = 0;
  Slot slots[kSlots];
  int next = 0;
};

DeviceWs g_ws[kMaxDevices];

int ensure_init(DeviceWs &ws) {
  if (ws.init) return RPA_OK;
  if (cudaMalloc(&ws.err, sizeof(uint32_t)) != cudaSuccess) return RPA_ERR_OOM;
  if (cudaMemset(ws.err, 0, sizeof(uint32_t)) != cudaSuccess) return RPA_ERR_CUDA;
  if (cudaEventCreateWithFlags(&ws.fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&ws.join, cudaEventDisableTiming) != cudaSuccess)
    return RPA_ERR_CUDA;
  for (auto &s : ws.slots)
    if (cudaEventCreateWithFlags(&s.done, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming) != cudaSuccess)
      return RPA_ERR_CUDA;
  // the side stream runs the prefill of a concurrent mixed batch: the
  // highest priority makes the block scheduler place its (whole-SM) CTAs
  // before the decode kernel's, which then fill each SM as it frees
  int lo_prio = 0, hi_prio = 0;
  if (cudaDeviceGetStreamPriorityRange(&lo_prio, &hi_prio) != cudaSuccess) hi_prio = 0;
  if (cudaStreamCreateWithPriority(&ws.side, cudaStreamNonBlocking, hi_prio) != cudaSuccess) return RPA_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&ws.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || ws.sms <= 0)
    ws.sms = 148;
  ws.init = true;
  return RPA_OK;
}

int grow_slot(Slot &s, int64_t words, int64_t partial_floats) {
  if (s.pending) {
    if (cudaEventSynchronize(s.done) != cudaSuccess) return RPA_ERR_CUDA;
    s.pending = false;
  }
  if (words > s.words) {
    int64_t w = std::max<int64_t>(words, 2 * s.words);
    w = std::max<int64_t>(w, 4096);
    if (s.host) cudaFreeHost(s.host);
    if (s.dev) cudaFree(s.dev);
    s.host = nullptr;
    s.dev = nullptr;
    s.words = 0;
    if (cudaMallocHost(&s.host, w * sizeof(int32_t)) != cudaSuccess) return RPA_ERR_OOM;
    if (cudaMalloc(&s.dev, w * sizeof(int32_t)) != cudaSuccess) return RPA_ERR_OOM;
    s.words = w;
  }
  if (partial_floats > s.partial_floats) {
    int64_t f = std::max<int64_t>(partial_floats, s.partial_floats + s.partial_floats / 2);
    if (s.partial) cudaFree(s.partial);
    s.partial = nullptr;
    s.partial_floats = 0;
    if (cudaMalloc(&s.partial, f * sizeof(float)) != cudaSuccess) return RPA_ERR_OOM;
    s.partial_floats = f;
  }
  return RPA_OK;
}

int plan_checked(const int32_t *cu, const int32_t *kv, int32_t n, const int32_t *dist,
                 const rpa_dims *d, HostPlan &hp) {
  int rc = validate_dims(d);
  if (rc) return rc;
  rc = validate_lengths(cu, kv, n, d);
  if (rc) return rc;
  if (n > 0) rc = validate_distribution(dist, cu, kv, n);
  if (rc) return rc;
  build_plan(cu, kv, n, dist, d, hp);
  return RPA_OK;
}


// ---------------------------------------------------------------- tracing
std::atomic<int32_t> g_profile_on{0};
std::mutex g_profile_mu;
struct Traced {
  int kind;
  cudaEvent_t a, b;
};
std::vector<Traced> g_traced;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Runs `launch` on `stream`, bracketed by events when tracing is on.
template <typename F>
cudaError_t traced(int kind, cudaStream_t stream, F &&launch) {
  if (!g_profile_on.load()) return launch();
  std::lock_guard<std::mutex> lock(g_profile_mu);
  Traced t{kind, take_event(), take_event()};
  if (!t.a || !t.b) return launch();
  cudaEventRecord(t.a, stream);
  cudaError_t e = launch();
  cudaEventRecord(t.b, stream);
  g_traced.push_back(t);
  return e;
}


// SMs for the prefill kernel of a batch with both kinds of rows when
// RPA_OPT_PREFILL_SMS is 0.  A decode SM moves a fixed share of HBM
// bandwidth and a prefill SM does a fixed share of the MMAs, so the step
// lasts about as long as the two kernels' summed SM-time over the GPU, and
// the schedule matters at the end: an SM that takes prefill units first and
// finishes them late, when the decode work is done, idles the rest.  So the
// prefill gets its estimated share of the SM-time (1.2 times it, even, at
// least 16 SMs) and the decode CTAs take the other SMs from the start.  The
// per-SM rates are this kernel set's measured ones on B200; only their ratio
// matters.
int auto_prefill_ctas(const HostPlan &hp, const Problem &pb, int sms) {
  constexpr double kPrefillFlopsPerSm128 = 6.0e12, kPrefillFlopsPerSm256 = 8.6e12;
  constexpr double kDecodeBytesPerSm = 41.0e9;
  double blocks = 0;   // 128-row x 128-key score blocks of every tile half (one query head)
  for (const PrefillTile &t : hp.prefill) {
    const int n_ctx = (t.kv_len - t.q_len + 127) / 128;
    for (int h = 0; h * 128 < t.rows; ++h) {
      const int rows = std::min(128, t.rows - h * 128);
      const int new_end = pb.causal ? t.tile_row + h * 128 + rows : t.q_len;
      blocks += n_ctx + (new_end + 127) / 128;
    }
  }
  const double flops = blocks * 128.0 * 128.0 * 4.0 * pb.d * pb.hq;
  double kv_blocks = 0;   // 16-token blocks of K/V read by the decode items
  for (const DecodeItem &it : hp.decode) kv_blocks += it.blk_end - it.blk_begin;
  for (const DecodeItem &it : hp.decode_packed) kv_blocks += it.blk_end - it.blk_begin;
  const double bytes = kv_blocks * 16.0 * pb.hkv * pb.d * 2.0 * 2.0;
  const double tp = flops / (pb.d > 128 ? kPrefillFlopsPerSm256 : kPrefillFlopsPerSm128);
  const double td = bytes / kDecodeBytesPerSm;
  if (tp <= 0 || td <= 0) return 0;
  int n = (int)std::ceil(1.2 * sms * tp / (tp + td));
  n = std::max(16, n + (n & 1));
  return n >= sms ? 0 : n;   // 0: one per SM
}

// The kernels of one planned call, queued on `stream` (the caller holds
// ws.mu).  A batch with both prefill and decode work runs them
// concurrently: the compute-bound prefill kernel on the high-priority side
// stream, queued first, takes the SMs (one whole-SM CTA each); the
// bandwidth-bound decode kernel on the caller's stream fills every SM its
// prefill CTA leaves, so the prefill's uneven finish is covered instead of
// waited for.  fork / join order the side stream against `stream`.
cudaError_t launch_kernels(DeviceWs &ws, const HostPlan &hp, const int32_t *dev_plan, float *partials,
                           Problem pb, cudaStream_t stream, cudaEvent_t fork, cudaEvent_t join) {
  pb.err = ws.err;
  const PlanLayout &L = hp.layout;
  const int G = pb.hq / pb.hkv;
  float *partial_o = partials;
  float *partial_lse = partials ? partials + L.n_partials * pb.hkv * G * pb.d : nullptr;
  cudaError_t e = cudaSuccess;
  const bool mixed = L.n_prefill_tiles > 0 &&
                     (L.n_decode_items > 0 || L.n_decode_packed > 0 || L.n_generic_rows > 0) &&
                     g_opt_concurrent_mixed.load() >= 0;
  cudaStream_t pstream = stream;
  int prefill_ctas = 0;
  if (mixed) {
    const int64_t k = g_opt_prefill_sms.load();
    prefill_ctas = k > 0 ? (int)std::min<int64_t>(k, ws.sms) : k == 0 ? auto_prefill_ctas(hp, pb, ws.sms) : 0;
    pstream = ws.side;
    if (cudaEventRecord(fork, stream) != cudaSuccess || cudaStreamWaitEvent(pstream, fork, 0) != cudaSuccess)
      return cudaErrorUnknown;
  }
  if (L.n_prefill_tiles > 0 && e == cudaSuccess)
    e = traced(RPA_KERNEL_PREFILL, pstream, [&] {
      const PrefillTile *tiles = (const PrefillTile *)(dev_plan + L.prefill_off);
      // context-heavy prefill (chunked rows after a long cache) gathers
      // latency-bound paged blocks and writes few new rows: a producer warp
      // per operand; fresh prefill keeps two warps for the cache update
      const int64_t lo = g_opt_prefill_loaders.load();
      const bool split = lo == 2 || (lo != 1 && hp.prefill_ctx_tokens > hp.prefill_new_tokens);
      return launch_prefill_any(pb, tiles, (int)L.n_prefill_tiles, prefill_ctas, split, pstream);
    });
  if (mixed && cudaEventRecord(join, pstream) != cudaSuccess) e = cudaErrorUnknown;
  if (L.n_decode_items > 0 && e == cudaSuccess)
    e = traced(RPA_KERNEL_DECODE, stream, [&] {
      return launch_decode(pb, (const DecodeItem *)(dev_plan + L.decode_off), (int)L.n_decode_items, partial_o,
                           partial_lse, false, stream);
    });
  if (L.n_decode_packed > 0 && e == cudaSuccess)
    e = traced(RPA_KERNEL_DECODE, stream, [&] {
      return launch_decode(pb, (const DecodeItem *)(dev_plan + L.decode_packed_off), (int)L.n_decode_packed,
                           partial_o, partial_lse, true, stream);
    });
  if (L.n_combine > 0 && e == cudaSuccess)
    e = traced(RPA_KERNEL_COMBINE, stream, [&] {
      // right behind the decode launch unless tracing events sit between them
      return launch_combine(pb, (const CombineItem *)(dev_plan + L.combine_off), (int)L.n_combine, partial_o,
                            partial_lse, stream, !g_profile_on.load());
    });
  if (L.n_generic_rows > 0 && e == cudaSuccess)
    e = traced(RPA_KERNEL_GENERIC, stream, [&] {
      return launch_generic(pb, (const GenericSeq *)(dev_plan + L.generic_off), (int)L.n_generic_seqs,
                            (int)L.n_generic_rows, stream);
    });
  // join: the caller's stream waits for the side stream (also on errors,
  // so that nothing of this call is left running unordered)
  if (mixed && cudaStreamWaitEvent(stream, join, 0) != cudaSuccess && e == cudaSuccess) e = cudaErrorUnknown;
  return e;
}

}  // namespace

int64_t plan_partial_floats(const HostPlan &hp, const rpa_dims &d) {
  return hp.layout.n_partials * (int64_t)d.num_q_heads * (d.head_dim + 1);
}

Problem problem_of(const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                   const int32_t *page_table, void *out, float *lse, const rpa_dims &d, float scale,
                   int32_t causal) {
  Problem pb{};
  pb.q = q;
  pb.k_new = k_new;
  pb.v_new = v_new;
  pb.k_cache = k_cache;
  pb.v_cache = v_cache;
  pb.page_table = page_table;
  pb.out = out;
  pb.lse = lse;
  pb.hq = d.num_q_heads;
  pb.hkv = d.num_kv_heads;
  pb.d = d.head_dim;
  pb.p = d.page_size;
  pb.num_pages = d.num_pages;
  pb.max_pages = d.max_pages_per_seq;
  pb.dtype = d.dtype;
  pb.causal = causal ? 1 : 0;
  pb.scale = scale;
  pb.total_q = d.total_q_tokens;
  return pb;
}

int launch_planned(const HostPlan &hp, const int32_t *dev_plan, float *partials, Problem pb,
                   cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RPA_ERR_CUDA;
  DeviceWs &ws = g_ws[dev];
  std::lock_guard<std::mutex> lock(ws.mu);
  const int rc = ensure_init(ws);
  if (rc) return rc;
  return launch_kernels(ws, hp, dev_plan, partials, pb, stream, ws.fork, ws.join) == cudaSuccess ? RPA_OK
                                                                                                  : RPA_ERR_CUDA;
}

}  // namespace rpa

using namespace rpa;

extern "C" RPA_API const char *rpa_status_string(int status) {
  switch (status) {
    case RPA_OK: return "ok";
    case RPA_ERR_INVALID_ARG: return "invalid argument";
    case RPA_ERR_UNSUPPORTED: return "unsupported geometry";
    case RPA_ERR_LENGTHS: return "invalid sequence lengths";
    case RPA_ERR_DISTRIBUTION: return "distribution inconsistent with lengths";
    case RPA_ERR_OOM: return "workspace allocation failed";
    case RPA_ERR_CUDA: return "CUDA error";
    case RPA_ERR_SCRATCH_LIMIT: return "batch exceeds the no-alloc scratch limit";
    case RPA_ERR_WORKSPACE: return "workspace too small or misaligned";
    default: return "unknown status";
  }
}

extern "C" RPA_API int64_t rpa_set_option(int32_t option, int64_t value) {
  switch (option) {
    case RPA_OPT_DECODE_CHUNK_BLOCKS: return g_opt_decode_chunk.exchange(value);
    case RPA_OPT_FORCE_GENERIC: return g_opt_force_generic.exchange(value);
    case RPA_OPT_DISABLE_PREFILL_TC: return g_opt_disable_prefill_tc.exchange(value);
    case RPA_OPT_PREFILL_SMS: return g_opt_prefill_sms.exchange(value);
    case RPA_OPT_CONCURRENT_MIXED: return g_opt_concurrent_mixed.exchange(value);
    case RPA_OPT_PREFILL_LOADERS: return g_opt_prefill_loaders.exchange(value);
    case RPA_OPT_DECODE_PACK_BLOCKS: return g_opt_decode_pack.exchange(value);
    case RPA_OPT_PREFILL_KERNEL: return g_opt_prefill_kernel.exchange(value);
    default: return -1;
  }
}

extern "C" RPA_API int rpa_plan(const int32_t *cu_q_lens, const int32_t *kv_lens, int32_t num_seqs,
                        const int32_t *distribution, const rpa_dims *dims, rpa_plan_info *info) {
  if (info == nullptr) return RPA_ERR_INVALID_ARG;
  try {
    HostPlan hp;
    int rc = plan_checked(cu_q_lens, kv_lens, num_seqs, distribution, dims, hp);
    if (rc) return rc;
    info->num_decode = hp.num_decode;
    info->num_prefill = hp.num_prefill;
    info->num_generic = hp.num_generic;
    info->num_empty = hp.num_empty;
    info->decode_items = (int32_t)(hp.decode.size() + hp.decode_packed.size());
    info->decode_packed = (int32_t)hp.decode_packed.size();
    info->decode_max_splits = hp.decode_max_splits;
    info->combine_rows = (int32_t)hp.combine.size();
    info->prefill_tiles = (int32_t)hp.prefill.size();
    info->plan_bytes = hp.layout.total_words * 4;
    return RPA_OK;
  } catch (const std::bad_alloc &) {
    return RPA_ERR_OOM;
  }
}

extern "C" RPA_API int rpa_forward(const void *q, const void *k_new, const void *v_new, void *k_cache,
                           void *v_cache, const int32_t *page_table, const int32_t *cu_q_lens,
                           const int32_t *kv_lens, int32_t num_seqs, const int32_t *distribution,
                           float scale, int32_t causal, void *out, float *lse,
                           const rpa_dims *dims, void *stream_ptr) {
  cudaStream_t stream = (cudaStream_t)stream_ptr;
  // the kernels take row maxima of the raw scores: the scale must be > 0
  if (!(scale > 0.f) || !std::isfinite(scale)) return RPA_ERR_INVALID_ARG;
  try {
    HostPlan hp;
    int rc = plan_checked(cu_q_lens, kv_lens, num_seqs, distribution, dims, hp);
    if (rc) return rc;
    const int32_t T = dims->total_q_tokens;
    if (num_seqs == 0 || T == 0) return RPA_OK;  // no new tokens: nothing to write or attend
    if (!q || !k_new || !v_new || !k_cache || !v_cache || !page_table || !out)
      return RPA_ERR_INVALID_ARG;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RPA_ERR_CUDA;
    DeviceWs &ws = g_ws[dev];
    std::lock_guard<std::mutex> lock(ws.mu);
    rc = ensure_init(ws);
    if (rc) return rc;
    Slot &slot = ws.slots[ws.next];
    ws.next = (ws.next + 1) % kSlots;

    const PlanLayout &L = hp.layout;
    if (L.n_prefill_tiles == 0 && L.n_generic_rows == 0 && L.n_decode_packed == 0 && L.n_decode_items > 0 &&
        decode_plan_fits_inline((int)L.n_decode_items, (int)L.n_combine)) {
      // A small decode-only batch: its work items and combine rows travel in
      // the launch parameters, with no plan copy ahead of the kernels.
      rc = grow_slot(slot, 0, plan_partial_floats(hp, *dims));
      if (rc) return rc;
      Problem pb = problem_of(q, k_new, v_new, k_cache, v_cache, page_table, out, lse, *dims, scale, causal);
      pb.err = ws.err;
      float *po = slot.partial;
      float *pl = po ? po + L.n_partials * (int64_t)dims->num_q_heads * dims->head_dim : nullptr;
      cudaError_t e = traced(RPA_KERNEL_DECODE, stream, [&] {
        return launch_decode_inline(pb, hp.decode.data(), (int)L.n_decode_items, po, pl, stream);
      });
      if (e == cudaSuccess && L.n_combine > 0)
        e = traced(RPA_KERNEL_COMBINE, stream, [&] {
          return launch_combine_inline(pb, hp.combine.data(), (int)L.n_combine, po, pl, stream, !g_profile_on.load());
        });
      if (cudaEventRecord(slot.done, stream) == cudaSuccess) slot.pending = true;
      return e == cudaSuccess ? RPA_OK : RPA_ERR_CUDA;
    }
    rc = grow_slot(slot, hp.layout.total_words, plan_partial_floats(hp, *dims));
    if (rc) return rc;
    serialize(hp, slot.host);
    if (hp.layout.total_words > 0 &&
        cudaMemcpyAsync(slot.dev, slot.host, hp.layout.total_words * sizeof(int32_t),
                        cudaMemcpyHostToDevice, stream) != cudaSuccess)
      return RPA_ERR_CUDA;
    Problem pb = problem_of(q, k_new, v_new, k_cache, v_cache, page_table, out, lse, *dims, scale, causal);
    const cudaError_t e = launch_kernels(ws, hp, slot.dev, slot.partial, pb, stream, slot.fork, slot.join);
    if (cudaEventRecord(slot.done, stream) == cudaSuccess) slot.pending = true;
    return e == cudaSuccess ? RPA_OK : RPA_ERR_CUDA;
  } catch (const std::bad_alloc &) {
    return RPA_ERR_OOM;
  }
}

extern "C" RPA_API int rpa_device_status(void *stream_ptr, uint32_t *flags) {
  if (flags == nullptr) return RPA_ERR_INVALID_ARG;
  *flags = 0;
  if (cudaStreamSynchronize((cudaStream_t)stream_ptr) != cudaSuccess) return RPA_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RPA_ERR_CUDA;
  DeviceWs &ws = g_ws[dev];
  std::lock_guard<std::mutex> lock(ws.mu);
  if (!ws.init) return RPA_OK;
  uint32_t v = 0;
  if (cudaMemcpy(&v, ws.err, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return RPA_ERR_CUDA;
  if (cudaMemset(ws.err, 0, sizeof v) != cudaSuccess) return RPA_ERR_CUDA;
  *flags = v;
  return RPA_OK;
}

extern "C" RPA_API int32_t rpa_profile_enable(int32_t on) { return g_profile_on.exchange(on ? 1 : 0); }

extern "C" RPA_API int rpa_profile_read(double *ms, int64_t *launches) {
  std::lock_guard<std::mutex> lock(g_profile_mu);
  double acc[RPA_KERNEL_CLASSES] = {0, 0, 0, 0};
  int64_t cnt[RPA_KERNEL_CLASSES] = {0, 0, 0, 0};
  int rc = RPA_OK;
  for (const Traced &t : g_traced) {
    float v = 0.f;
    if (cudaEventSynchronize(t.b) != cudaSuccess || cudaEventElapsedTime(&v, t.a, t.b) != cudaSuccess)
      rc = RPA_ERR_CUDA;
    acc[t.kind] += v;
    cnt[t.kind] += 1;
    g_event_pool.push_back(t.a);
    g_event_pool.push_back(t.b);
  }
  g_traced.clear();
  for (int k = 0; k < RPA_KERNEL_CLASSES; ++k) {
    if (ms) ms[k] = acc[k];
    if (launches) launches[k] = cnt[k];
  }
  return rc;
}
