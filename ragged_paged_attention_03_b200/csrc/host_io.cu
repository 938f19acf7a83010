// host_io.cu -- rpa_forward_host: the attention pass for a caller whose new
// tokens' q / k_new / v_new, page table and results live in host memory,
// with the PCIe copies overlapped with the kernels.
//
// The batch is cut into groups of whole, consecutive sequences (a group's
// tokens are one contiguous row range of q / k_new / v_new / out / lse, its
// page-table rows one contiguous range), and each group is planned by
// rpa_forward's planner.  On the host-to-device copy stream: the page table
// and the first group's inputs (queued before the planning, so the copy
// engine starts at once), then all groups' plans in one copy, then the other
// groups' inputs.  Each group's kernels (rpa_forward's) wait only for their
// own inputs, and its results go back as soon as it is done.  Groups of
// decode sequences only (long kernels, few bytes) run on the caller's
// stream, the others on a high-priority compute stream, each kind with its
// own copy-back stream, so that a long decode group neither holds up the
// kernels of the prefill groups behind it nor their results.
// A step then costs about its input transfer time plus the last group's
// compute and result copy, instead of the sum of all three.  Attention of
// one sequence never reads another's rows, so the grouping does not change
// what is computed; it changes the per-group work split (decode split-KV
// chunking) and hence the fp32 summation order only.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <vector>

#include "forward_internal.h"
#include "host_common.h"
#include "rpa.h"

namespace rpa {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxGroups = RPA_HOST_MAX_GROUPS;
// Below this many bytes of copies a step is one group: the copies take a few
// microseconds, and splitting the batch would only shrink each launch.
constexpr int64_t kPipelineMinBytes = 8ll << 20;
// Smallest group a pipelined step aims for (per-copy overhead stays small).
constexpr int64_t kGroupMinBytes = 4ll << 20;

struct Sizes {
  int64_t in_tok;    // q + k_new + v_new bytes of one new token
  int64_t out_tok;   // out (+ lse) bytes of one new token
  int64_t q_tok, kv_tok, o_tok, lse_tok;
};

Sizes sizes_of(const rpa_dims &d, bool with_lse) {
  const int64_t e = d.dtype == RPA_BF16 ? 2 : 4;
  Sizes s;
  s.q_tok = (int64_t)d.num_q_heads * d.head_dim * e;
  s.kv_tok = (int64_t)d.num_kv_heads * d.head_dim * e;
  s.o_tok = s.q_tok;
  s.lse_tok = with_lse ? (int64_t)d.num_q_heads * 4 : 0;
  s.in_tok = s.q_tok + 2 * s.kv_tok;
  s.out_tok = s.o_tok + s.lse_tok;
  return s;
}

// Group boundaries (sequence indices, bounds[0] = 0, bounds[n] = num_seqs).
// A group takes sequences in order until the next one would carry it past
// the target size; the target is a sixteenth of the step's bytes, at least
// kGroupMinBytes.  "Would carry it past" (not "has reached") keeps a run of
// small sequences (decode) apart from a large one that follows, so their
// long, copy-light attention starts while the large inputs are in flight.
int make_groups(const int32_t *cu, int32_t n, const Sizes &sz, int32_t *bounds) {
  const int64_t per_tok = sz.in_tok + sz.out_tok;
  const int64_t total = (int64_t)cu[n] * per_tok;
  bounds[0] = 0;
  if (total < kPipelineMinBytes || n <= 1) {
    bounds[1] = n;
    return 1;
  }
  const int64_t target = std::max<int64_t>(kGroupMinBytes, (total + 15) / 16);
  int g = 0;
  int64_t cur = 0;
  for (int32_t s = 0; s < n; ++s) {
    const int64_t b = (int64_t)(cu[s + 1] - cu[s]) * per_tok;
    if (cur > 0 && cur + b > target && g + 1 < kMaxGroups) {
      bounds[++g] = s;
      cur = 0;
    }
    cur += b;
  }
  bounds[++g] = n;
  return g;
}

// Page-locked staging of one call's plans.  Two alternate, so that a call
// waits (on the host) only for the plan copy of the call before the last.
struct PinnedPlan {
  int32_t *host = nullptr;
  int64_t words = 0;
  cudaEvent_t copied = nullptr;   // recorded after the plan copy
  bool pending = false;
};

// A growable device buffer that an earlier call may still be using.
struct DevBuf {
  unsigned char *ptr = nullptr;
  int64_t bytes = 0;
};

// Per device: the copy and compute streams, the events that order them
// against the caller's stream, the device staging of a call's inputs and
// results (q | k_new | v_new | out | lse | page table), the device plans and
// split-KV partials, and the pinned plan staging.
struct HostIo {
  std::mutex mu;
  bool init = false;
  cudaStream_t h2d = nullptr;
  cudaStream_t comp_hi = nullptr;             // groups with prefill rows
  cudaStream_t d2h = nullptr, d2h_hi = nullptr;   // results of decode groups / of the others
  cudaEvent_t fork = nullptr, join[3] = {}, done = nullptr;
  cudaEvent_t in[kMaxGroups] = {}, comp[kMaxGroups] = {};
  bool done_pending = false;   // `done` was recorded by an earlier call
  DevBuf io, plan;
  PinnedPlan pin[2];
  int next_pin = 0;
};

HostIo g_io[kMaxDevices];

int ensure_init(HostIo &io) {
  if (io.init) return RPA_OK;
  int lo_prio = 0, hi_prio = 0;
  if (cudaDeviceGetStreamPriorityRange(&lo_prio, &hi_prio) != cudaSuccess) hi_prio = 0;
  if (cudaStreamCreateWithFlags(&io.h2d, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithPriority(&io.comp_hi, cudaStreamNonBlocking, hi_prio) != cudaSuccess ||
      cudaStreamCreateWithFlags(&io.d2h, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&io.d2h_hi, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&io.fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&io.done, cudaEventDisableTiming) != cudaSuccess)
    return RPA_ERR_CUDA;
  for (auto &e : io.join)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return RPA_ERR_CUDA;
  for (auto &p : io.pin)
    if (cudaEventCreateWithFlags(&p.copied, cudaEventDisableTiming) != cudaSuccess) return RPA_ERR_CUDA;
  for (int g = 0; g < kMaxGroups; ++g)
    if (cudaEventCreateWithFlags(&io.in[g], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&io.comp[g], cudaEventDisableTiming) != cudaSuccess)
      return RPA_ERR_CUDA;
  io.init = true;
  return RPA_OK;
}

int64_t align256(int64_t x) { return (x + 255) & ~(int64_t)255; }

struct Staging {
  int64_t q, kn, vn, out, lse, pt, total;
};

Staging staging_of(const rpa_dims &d, const Sizes &sz, int32_t n) {
  const int64_t T = d.total_q_tokens;
  Staging st;
  st.q = 0;
  st.kn = st.q + align256(T * sz.q_tok);
  st.vn = st.kn + align256(T * sz.kv_tok);
  st.out = st.vn + align256(T * sz.kv_tok);
  st.lse = st.out + align256(T * sz.o_tok);
  st.pt = st.lse + align256(T * sz.lse_tok);
  st.total = st.pt + align256((int64_t)n * d.max_pages_per_seq * 4);
  return st;
}

// Grows `b` to at least `need` bytes.  The previous call's copies and
// kernels may still use the old buffer: its `done` event is waited for first.
int grow(HostIo &io, DevBuf &b, int64_t need) {
  if (need <= b.bytes) return RPA_OK;
  if (io.done_pending && cudaEventSynchronize(io.done) != cudaSuccess) return RPA_ERR_CUDA;
  io.done_pending = false;
  const int64_t nb = std::max<int64_t>(need, b.bytes + b.bytes / 2);
  if (b.ptr) cudaFree(b.ptr);
  b.ptr = nullptr;
  b.bytes = 0;
  if (cudaMalloc(&b.ptr, nb) != cudaSuccess) return RPA_ERR_OOM;
  b.bytes = nb;
  return RPA_OK;
}

int grow_pinned(PinnedPlan &p, int64_t words) {
  // the plan copy that last read this buffer must have run
  if (p.pending && cudaEventSynchronize(p.copied) != cudaSuccess) return RPA_ERR_CUDA;
  p.pending = false;
  if (words <= p.words) return RPA_OK;
  const int64_t w = std::max<int64_t>(std::max<int64_t>(words, 2 * p.words), 16384);
  if (p.host) cudaFreeHost(p.host);
  p.host = nullptr;
  p.words = 0;
  if (cudaMallocHost(&p.host, w * 4) != cudaSuccess) return RPA_ERR_OOM;
  p.words = w;
  return RPA_OK;
}

}  // namespace
}  // namespace rpa

using namespace rpa;

extern "C" RPA_API int rpa_host_groups(const int32_t *cu_q_lens, int32_t num_seqs, const rpa_dims *dims,
                                       int32_t with_lse, int32_t *bounds, int32_t *num_groups) {
  if (bounds == nullptr || num_groups == nullptr) return RPA_ERR_INVALID_ARG;
  *num_groups = 0;
  int rc = validate_dims(dims);
  if (rc) return rc;
  if (num_seqs < 0) return RPA_ERR_INVALID_ARG;
  if (num_seqs == 0) {
    bounds[0] = 0;
    return RPA_OK;
  }
  if (cu_q_lens == nullptr) return RPA_ERR_INVALID_ARG;
  if (cu_q_lens[0] != 0 || cu_q_lens[num_seqs] != dims->total_q_tokens) return RPA_ERR_LENGTHS;
  for (int32_t s = 0; s < num_seqs; ++s)
    if (cu_q_lens[s + 1] < cu_q_lens[s]) return RPA_ERR_LENGTHS;
  *num_groups = make_groups(cu_q_lens, num_seqs, sizes_of(*dims, with_lse != 0), bounds);
  return RPA_OK;
}

extern "C" RPA_API int rpa_forward_host(const void *q, const void *k_new, const void *v_new, void *k_cache,
                                        void *v_cache, const int32_t *page_table, const int32_t *cu_q_lens,
                                        const int32_t *kv_lens, int32_t num_seqs, const int32_t *distribution,
                                        float scale, int32_t causal, void *out, float *lse,
                                        const rpa_dims *dims, void *stream_ptr) {
  cudaStream_t stream = (cudaStream_t)stream_ptr;
  if (!(scale > 0.f) || !std::isfinite(scale)) return RPA_ERR_INVALID_ARG;
  int rc = validate_dims(dims);
  if (rc) return rc;
  rc = validate_lengths(cu_q_lens, kv_lens, num_seqs, dims);
  if (rc) return rc;
  if (num_seqs > 0) rc = validate_distribution(distribution, cu_q_lens, kv_lens, num_seqs);
  if (rc) return rc;
  const int32_t T = dims->total_q_tokens;
  if (num_seqs == 0 || T == 0) return RPA_OK;
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !page_table || !out) return RPA_ERR_INVALID_ARG;

  try {
    const Sizes sz = sizes_of(*dims, lse != nullptr);
    int32_t bounds[kMaxGroups + 1];
    const int ng = make_groups(cu_q_lens, num_seqs, sz, bounds);
    const int64_t mp = dims->max_pages_per_seq;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RPA_ERR_CUDA;
    HostIo &io = g_io[dev];
    std::lock_guard<std::mutex> lock(io.mu);
    rc = ensure_init(io);
    if (rc) return rc;
    const Staging st = staging_of(*dims, sz, num_seqs);
    rc = grow(io, io.io, st.total);
    if (rc) return rc;
    unsigned char *b = io.io.ptr;
    std::vector<HostPlan> plans(ng);
    std::vector<int64_t> plan_off(ng + 1, 0), part_off(ng + 1, 0);
    std::vector<int32_t> cu_g(num_seqs + 1);
    std::vector<char> has_prefill(ng, 0);

    // One group has nothing to overlap: everything runs on the caller's
    // stream, in order, without the event hops between streams.  Otherwise
    // the copy and compute streams start after the caller's earlier work
    // (which may have filled the host inputs).  Both wait for the previous
    // call of this function on any stream (which may still use the staging
    // buffers).
    const bool one = ng == 1;
    cudaStream_t h2d = one ? stream : io.h2d;
    cudaError_t e = cudaSuccess;
    if (one) {
      if (io.done_pending) e = cudaStreamWaitEvent(stream, io.done, 0);
    } else {
      cudaStream_t side[4] = {io.h2d, io.comp_hi, io.d2h, io.d2h_hi};
      e = cudaEventRecord(io.fork, stream);
      for (cudaStream_t sd : side) {
        if (e == cudaSuccess) e = cudaStreamWaitEvent(sd, io.fork, 0);
        if (e == cudaSuccess && io.done_pending) e = cudaStreamWaitEvent(sd, io.done, 0);
      }
    }
    auto copy_in = [&](int g) {
      const int64_t t0 = cu_q_lens[bounds[g]], nt = cu_q_lens[bounds[g + 1]] - t0;
      cudaError_t r = cudaSuccess;
      if (nt > 0) {
        r = cudaMemcpyAsync(b + st.q + t0 * sz.q_tok, (const unsigned char *)q + t0 * sz.q_tok, nt * sz.q_tok,
                            cudaMemcpyHostToDevice, h2d);
        if (r == cudaSuccess)
          r = cudaMemcpyAsync(b + st.kn + t0 * sz.kv_tok, (const unsigned char *)k_new + t0 * sz.kv_tok,
                              nt * sz.kv_tok, cudaMemcpyHostToDevice, h2d);
        if (r == cudaSuccess)
          r = cudaMemcpyAsync(b + st.vn + t0 * sz.kv_tok, (const unsigned char *)v_new + t0 * sz.kv_tok,
                              nt * sz.kv_tok, cudaMemcpyHostToDevice, h2d);
      }
      return r;
    };
    // the page table and the first group's inputs go in while the host plans
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(b + st.pt, page_table, (size_t)num_seqs * mp * 4, cudaMemcpyHostToDevice, h2d);
    if (e == cudaSuccess) e = copy_in(0);

    // ---- plan every group (rpa_forward's planner on the group's lengths,
    // token rows and page-table rows counted from the group start).  Copies
    // are queued already: a failed host allocation from here on still ends
    // with the streams joined below.
    try {
      for (int g = 0; g < ng; ++g) {
        const int32_t s0 = bounds[g], ns = bounds[g + 1] - bounds[g];
        const int32_t t0 = cu_q_lens[s0];
        for (int32_t s = 0; s <= ns; ++s) {
          cu_g[s] = cu_q_lens[s0 + s] - t0;
          if (s > 0 && cu_g[s] - cu_g[s - 1] > 1) has_prefill[g] = 1;
        }
        int32_t dist_g[3];
        const int32_t *dist_p = nullptr;
        if (distribution) {
          for (int i = 0; i < 2; ++i) dist_g[i] = std::min(std::max(distribution[i], s0), s0 + ns) - s0;
          dist_g[2] = ns;
          dist_p = dist_g;
        }
        rpa_dims dg = *dims;
        dg.total_q_tokens = cu_g[ns];
        build_plan(cu_g.data(), kv_lens + s0, ns, dist_p, &dg, plans[g]);
        plan_off[g + 1] = plan_off[g] + ((plans[g].layout.total_words + 63) & ~(int64_t)63);   // 256-byte steps
        // groups may run concurrently: each has its own partials
        part_off[g + 1] = part_off[g] + ((plan_partial_floats(plans[g], dg) + 63) & ~(int64_t)63);
      }
    } catch (const std::bad_alloc &) {
      rc = RPA_ERR_OOM;
    }
    const int64_t plan_words = plan_off[ng];
    if (e == cudaSuccess && rc == RPA_OK) rc = grow(io, io.plan, plan_words * 4 + part_off[ng] * 4);
    PinnedPlan &pin = io.pin[io.next_pin];
    io.next_pin ^= 1;
    if (e == cudaSuccess && rc == RPA_OK) rc = grow_pinned(pin, plan_words);
    const int32_t *dplan = (const int32_t *)io.plan.ptr;
    float *dpart = (float *)(io.plan.ptr + plan_words * 4);
    if (e == cudaSuccess && rc == RPA_OK) {
      for (int g = 0; g < ng; ++g) serialize(plans[g], pin.host + plan_off[g]);
      if (plan_words > 0)
        e = cudaMemcpyAsync(io.plan.ptr, pin.host, plan_words * 4, cudaMemcpyHostToDevice, h2d);
      if (e == cudaSuccess && cudaEventRecord(pin.copied, h2d) == cudaSuccess) pin.pending = true;
      if (e == cudaSuccess && !one) e = cudaEventRecord(io.in[0], h2d);
      for (int g = 1; g < ng && e == cudaSuccess; ++g) {
        e = copy_in(g);
        if (e == cudaSuccess) e = cudaEventRecord(io.in[g], h2d);
      }
    }

    // per group: its kernels, then its results back
    for (int g = 0; g < ng && e == cudaSuccess && rc == RPA_OK; ++g) {
      const int32_t s0 = bounds[g];
      const int64_t t0 = cu_q_lens[s0], nt = cu_q_lens[bounds[g + 1]] - t0;
      if (nt == 0) continue;   // only q_len = 0 sequences: nothing to write or read back
      // RPA_OPT_CONCURRENT_MIXED < 0: every group's kernels in order on the
      // caller's stream (as rpa_forward then runs prefill and decode serially)
      const bool side = !one && has_prefill[g] && concurrent_mixed();
      cudaStream_t cs = side ? io.comp_hi : stream;
      cudaStream_t os = one ? stream : side ? io.d2h_hi : io.d2h;
      rpa_dims dg = *dims;
      dg.total_q_tokens = (int32_t)nt;
      if (!one) e = cudaStreamWaitEvent(cs, io.in[g], 0);
      if (e != cudaSuccess) break;
      const Problem pb = problem_of(b + st.q + t0 * sz.q_tok, b + st.kn + t0 * sz.kv_tok, b + st.vn + t0 * sz.kv_tok,
                                    k_cache, v_cache, (const int32_t *)(b + st.pt) + (int64_t)s0 * mp,
                                    b + st.out + t0 * sz.o_tok,
                                    lse ? (float *)(b + st.lse) + t0 * dims->num_q_heads : nullptr, dg, scale,
                                    causal);
      rc = launch_planned(plans[g], dplan + plan_off[g], dpart + part_off[g], pb, cs);
      if (rc != RPA_OK) break;
      if (!one) e = cudaEventRecord(io.comp[g], cs);
      if (e == cudaSuccess && !one) e = cudaStreamWaitEvent(os, io.comp[g], 0);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync((unsigned char *)out + t0 * sz.o_tok, b + st.out + t0 * sz.o_tok, nt * sz.o_tok,
                            cudaMemcpyDeviceToHost, os);
      if (e == cudaSuccess && lse)
        e = cudaMemcpyAsync(lse + t0 * dims->num_q_heads, (float *)(b + st.lse) + t0 * dims->num_q_heads,
                            nt * sz.lse_tok, cudaMemcpyDeviceToHost, os);
    }
    // join: the caller's stream waits for every other stream of the call
    // (also after an error, so that nothing of the call is left running
    // unordered); `done`, recorded after the join, covers all of it
    cudaError_t ej = cudaSuccess;
    if (!one) {
      cudaStream_t joined[3] = {io.h2d, io.comp_hi, io.d2h_hi};
      for (int i = 0; i < 3 && ej == cudaSuccess; ++i) {
        ej = cudaEventRecord(io.join[i], joined[i]);
        if (ej == cudaSuccess) ej = cudaStreamWaitEvent(stream, io.join[i], 0);
      }
      if (ej == cudaSuccess) ej = cudaEventRecord(io.fork, io.d2h);
      if (ej == cudaSuccess) ej = cudaStreamWaitEvent(stream, io.fork, 0);
    }
    if (ej == cudaSuccess) ej = cudaEventRecord(io.done, stream);
    if (ej == cudaSuccess) io.done_pending = true;
    if (rc != RPA_OK) return rc;
    if (e != cudaSuccess || ej != cudaSuccess) return RPA_ERR_CUDA;
    return RPA_OK;
  } catch (const std::bad_alloc &) {
    return RPA_ERR_OOM;
  }
}
