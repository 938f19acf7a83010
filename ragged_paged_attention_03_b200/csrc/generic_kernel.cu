// generic_kernel.cu -- the simple, any-shape SIMT path.
//
// One warp per (query row, query head).  It walks the visible keys of its
// row in order, keeping a running max and sum (online softmax, the
// FlashAttention recurrence named in the RPA talk summary's glossary), and
// reads each key from its cache page (context positions) or from k_new (the
// row's own sequence's new tokens), never from a cache slot this call writes.
// The warps of query heads h with h % G == 0 also store their token's new
// K/V into its cache slot: the fused cache update of the talk summary,
// 00:06:36, with no separate scatter launch.
//
// This path carries fp32 (where tensor cores would round) and any shape the
// specialised kernels do not take; it is not tuned for speed.
#include <cuda_bf16.h>
#include <math.h>

#include "kernels.h"

namespace rpa {
namespace {

template <typename T>
struct Vec;  // D/32 contiguous elements per lane, loaded as wide as possible

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float v, float *p) { *p = v; }
__device__ __forceinline__ void from_f(float v, __nv_bfloat16 *p) { *p = __float2bfloat16_rn(v); }

template <typename T, int D>
__global__ void __launch_bounds__(128) generic_kernel(Problem pb, const GenericSeq *seqs,
                                                      int n_seqs, int n_rows) {
  constexpr int E = D / 32;  // elements per lane
  const int lane = threadIdx.x & 31;
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (pb.dev_counts != nullptr) {
    n_seqs = min(n_seqs, pb.dev_counts[kCntGenericSeqs]);
    n_rows = min(n_rows, pb.dev_counts[kCntGenericRows]);
  }
  if (warp >= (long long)n_rows * pb.hq) return;
  const int row = (int)(warp / pb.hq);
  const int h = (int)(warp % pb.hq);

  // the generic sequence that owns this row (largest row_prefix <= row)
  int lo = 0, hi = n_seqs - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (seqs[mid].row_prefix <= row) lo = mid; else hi = mid - 1;
  }
  const GenericSeq gs = seqs[lo];
  const int i = row - gs.row_prefix;        // new-token index within the sequence
  const int t = gs.q_start + i;             // global token row
  const int c = gs.kv_len - gs.q_len;       // cached context length
  const int G = pb.hq / pb.hkv;
  const int hk = h / G;
  const T *q = (const T *)pb.q;
  const T *kn = (const T *)pb.k_new;
  const T *vn = (const T *)pb.v_new;
  T *kc = (T *)pb.k_cache;
  T *vc = (T *)pb.v_cache;
  const int32_t *pt_row = pb.page_table + (size_t)gs.seq * pb.max_pages;

  // fused cache update of this token's K/V for KV head hk
  if (kCacheWrite && h % G == 0) {
    const int pos = c + i;
    const int page = pt_row[pos / pb.p];
    if (page >= 0 && page < pb.num_pages) {
      size_t dst = (((size_t)page * pb.p + pos % pb.p) * pb.hkv + hk) * D;
      size_t src = ((size_t)t * pb.hkv + hk) * D;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        kc[dst + lane * E + e] = kn[src + lane * E + e];
        vc[dst + lane * E + e] = vn[src + lane * E + e];
      }
    } else if (lane == 0) {
      atomicOr(pb.err, RPA_DEV_BAD_PAGE);
    }
  }

  float qv[E], acc[E];
  const size_t qoff = ((size_t)t * pb.hq + h) * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qv[e] = to_f(q[qoff + e]);
    acc[e] = 0.f;
  }
  const int nvis = pb.causal ? c + i + 1 : gs.kv_len;
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j < nvis; ++j) {
    const T *kp;
    const T *vp;
    bool ok = true;
    if (j < c) {
      const int page = pt_row[j / pb.p];
      ok = page >= 0 && page < pb.num_pages;
      size_t off = (((size_t)(ok ? page : 0) * pb.p + j % pb.p) * pb.hkv + hk) * D;
      kp = kc + off;
      vp = vc + off;
      if (!ok && lane == 0) atomicOr(pb.err, RPA_DEV_BAD_PAGE);
    } else {
      size_t off = ((size_t)(gs.q_start + j - c) * pb.hkv + hk) * D;
      kp = kn + off;
      vp = vn + off;
    }
    float kv[E], vv[E];
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      kv[e] = ok ? to_f(kp[lane * E + e]) : 0.f;
      vv[e] = ok ? to_f(vp[lane * E + e]) : 0.f;
      dot = fmaf(qv[e], kv[e], dot);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    const float s = dot * pb.scale;
    const float m_new = fmaxf(m, s);
    const float alpha = expf(m - m_new);   // 0 on the first key (m = -inf)
    const float p = expf(s - m_new);
    l = l * alpha + p;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = fmaf(p, vv[e], acc[e] * alpha);
    m = m_new;
  }
  T *out = (T *)pb.out;
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < E; ++e) from_f(acc[e] * inv, &out[qoff + e]);
  if (pb.lse != nullptr && lane == 0) pb.lse[(size_t)t * pb.hq + h] = m + logf(l);
}

template <typename T>
cudaError_t launch_t(const Problem &pb, const GenericSeq *seqs, int n_seqs, int n_rows,
                     cudaStream_t stream) {
  long long warps = (long long)n_rows * pb.hq;
  unsigned blocks = (unsigned)((warps + 3) / 4);
  switch (pb.d) {
    case 64: generic_kernel<T, 64><<<blocks, 128, 0, stream>>>(pb, seqs, n_seqs, n_rows); break;
    case 128: generic_kernel<T, 128><<<blocks, 128, 0, stream>>>(pb, seqs, n_seqs, n_rows); break;
    case 256: generic_kernel<T, 256><<<blocks, 128, 0, stream>>>(pb, seqs, n_seqs, n_rows); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_generic(const Problem &pb, const GenericSeq *seqs, int n_seqs, int n_rows,
                           cudaStream_t stream) {
  if (n_rows <= 0) return cudaSuccess;
  return pb.dtype == RPA_F32 ? launch_t<float>(pb, seqs, n_seqs, n_rows, stream)
                             : launch_t<__nv_bfloat16>(pb, seqs, n_seqs, n_rows, stream);
}

}  // namespace rpa
