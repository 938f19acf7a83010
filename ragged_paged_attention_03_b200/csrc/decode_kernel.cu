// decode_kernel.cu -- bandwidth-bound decode attention (one new token per
// sequence) with the fused cache update, plus the split-KV LSE combine.
//
// The RPA pages describe decode as bound by memory bandwidth (talk summary,
// 00:08:21: bandwidth saturates only from ~8K context tokens at head_dim 128)
// and hide the cache write behind the attention (00:06:36).  The B200 design:
//
// * One CTA per (work item, KV head).  A work item is a chunk of 16-token
//   blocks of one sequence; long sequences are cut into several items whose
//   partial results the combine kernel merges (log-sum-exp weighting).
// * Short sequences are packed instead: four whole-sequence items per CTA,
//   one per warp, each warp streaming all of its item's blocks (the
//   multi-request batching the talk's roadmap, 00:18:14, proposes for
//   sequences too short to fill the bandwidth on their own).
// * The CTA's four warps stream disjoint blocks (block b goes to warp
//   b mod 4), each with its own ring of shared-memory stages fed by TMA
//   (cp.async.bulk.tensor, 128-byte swizzle, one 16-row box per page part
//   and 64-column half).  No warp ever waits for another until the merge.
// * The G query heads of the KV head form the N side of a swap-AB MMA:
//   S^T[16 tokens x 8 heads] = K Q^T, then O^T[D x 8] += V^T P^T, with P^T
//   moved into the B-operand layout by movmatrix.  Tensor cores are used here
//   only to cut instruction issue per byte; the kernel stays HBM-bound.
// * Online softmax in the log2 domain with warp shuffles; the four warps'
//   (m, l, O) are merged through shared memory at the end.
// * The block holding position kv_len - 1 takes that row from k_new / v_new
//   instead of the cache (rows past it are zeroed), and the warp that owns
//   it stores the new K/V into the cache slot: exactly one writer per
//   (sequence, KV head), and nobody reads that slot from the cache.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <string.h>

#include "kernels.h"
#include "ptx.cuh"
#include "tma.h"

namespace rpa {
namespace {

constexpr int kWarps = 4;
constexpr int kMaxItemPages = 1024;   // page-table entries one work item may touch
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct DecodeShape {
  static constexpr int kHalves = D / 64;                  // 128-byte column tiles
  static constexpr int kTile = 16 * 128;                  // 16 rows x 64 bf16, swizzled
  static constexpr int kStage = 2 * kHalves * kTile;      // K tiles then V tiles
  static constexpr int kStages = D == 64 ? 6 : (D == 128 ? 2 : 3);
  static constexpr int kRing = kWarps * kStages * kStage;
  static constexpr int kSmem = 1024 + kRing + kMaxItemPages * 4 + kWarps * kStages * 8;
};

// Byte offset of (row r, 16-byte chunk ch) inside a stage's K or V part:
// column tile ch / 8, swizzled chunk (ch % 8) ^ (r % 8).
__device__ __forceinline__ uint32_t tile_off(int r, int ch) {
  return (uint32_t)((ch >> 3) * (16 * 128) + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

// PACK: each warp takes a whole work item of its own (item blockIdx.x * 4 +
// warp) -- short sequences, several per CTA -- and writes its result from
// registers; otherwise the four warps share one item and merge at the end.
template <int D, int NG, bool PACK>
__device__ __forceinline__ void decode_body(const CUtensorMap &tm_k, const CUtensorMap &tm_v, const Problem &pb,
                                            const DecodeItem *__restrict__ items, int n_items,
                                            float *__restrict__ part_o, float *__restrict__ part_lse,
                                            float scale_log2) {
  using S = DecodeShape<D>;
  // a split-KV combine queued behind this grid may be scheduled as soon as
  // every CTA of it has started; it waits for this grid's results itself
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int NST = S::kStages;
  constexpr int KS = D / 16;  // k-steps of QK^T, m-tiles of PV
  extern __shared__ uint8_t smem_raw[];
  uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int32_t *pages = reinterpret_cast<int32_t *>(ring + S::kRing);
  uint64_t *bars = reinterpret_cast<uint64_t *>(pages + kMaxItemPages);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (pb.dev_counts != nullptr) n_items = min(n_items, pb.dev_counts[PACK ? kCntPacked : kCntDecode]);
  // capacity-sized grid of a device-planned call: CTAs past the work leave
  if ((PACK ? (int)blockIdx.x * kWarps : (int)blockIdx.x) >= n_items) return;
  const int item_idx = PACK ? (int)blockIdx.x * kWarps + warp : (int)blockIdx.x;
  const bool has_item = item_idx < n_items;   // PACK: the last CTA may hold fewer items
  DecodeItem it = items[has_item ? item_idx : 0];
  if (!has_item) it.blk_begin = it.blk_end = 0;
  const int hk = blockIdx.y;
  const int G = pb.hq / pb.hkv;
  const int kv = it.kv_len;
  const int c = kv - 1;                       // cached positions are [0, c)
  const int P = pb.p;
  const int nblk_total = (kv + 15) >> 4;      // the last block holds position c
  const int first_page = (it.blk_begin * 16) / P;
  const int last_page = (min(it.blk_end * 16, kv) - 1) / P;
  const int npg = has_item ? last_page - first_page + 1 : 0;
  const int32_t *pt_row = pb.page_table + (size_t)it.seq * pb.max_pages;
  // PACK: a quarter of the page slots per warp
  int32_t *my_pages = pages + (PACK ? warp * (kMaxItemPages / kWarps) : 0);

  if (tid == 0) {
    ptx::tma_prefetch_desc(&tm_k);
    ptx::tma_prefetch_desc(&tm_v);
  }
  for (int i = PACK ? lane : tid; i < npg; i += PACK ? 32 : (int)blockDim.x) {
    int pg = pt_row[first_page + i];
    if (pg < 0 || pg >= pb.num_pages) {
      atomicOr(pb.err, RPA_DEV_BAD_PAGE);
      pg = -1;
    }
    my_pages[i] = pg;
  }
  if (tid < kWarps * NST) ptx::mbar_init(&bars[tid], 1);
  ptx::fence_barrier_init();
  __syncthreads();

  uint8_t *my_ring = ring + warp * NST * S::kStage;
  uint64_t *my_bars = bars + warp * NST;
  const int box_rows = P < 16 ? P : 16;

  // Queues the TMA copies of this warp's it-th block into its stage
  // (lane 0 only).  Boxes holding no cached position are skipped; their rows
  // are filled when the block is consumed.
  // every K/V byte is read by this CTA alone, once: first out of L2, so that
  // a prefill kernel running beside it keeps its reused K/V blocks there
  const uint64_t once = ptx::l2_evict_first_policy();
  auto issue = [&](int k) {
    const int b = it.blk_begin + (PACK ? k : warp + kWarps * k);
    if (b >= it.blk_end) return;
    const int st = k % NST;
    uint8_t *sk = my_ring + st * S::kStage;
    uint8_t *sv = sk + S::kHalves * S::kTile;
    uint32_t bytes = 0;
    for (int r0 = 0; r0 < 16; r0 += box_rows) {
      const int pos = b * 16 + r0;
      if (pos < c && my_pages[pos / P - first_page] >= 0) bytes += 2u * S::kHalves * 128u * box_rows;
    }
    if (bytes == 0) {
      ptx::mbar_arrive(&my_bars[st]);
      return;
    }
    ptx::mbar_arrive_expect_tx(&my_bars[st], bytes);
    for (int r0 = 0; r0 < 16; r0 += box_rows) {
      const int pos = b * 16 + r0;
      if (pos >= c) break;
      const int pg = my_pages[pos / P - first_page];
      if (pg < 0) continue;
      const int row = pg * P + (pos % P);
#pragma unroll
      for (int h = 0; h < S::kHalves; ++h) {
        ptx::tma_load_3d_hint(sk + h * S::kTile + r0 * 128, &tm_k, &my_bars[st], h * 64, hk, row, once);
        ptx::tma_load_3d_hint(sv + h * S::kTile + r0 * 128, &tm_v, &my_bars[st], h * 64, hk, row, once);
      }
    }
  };

  if (lane == 0)
    for (int k = 0; k < NST; ++k) issue(k);

  // Q^T fragments (B operand, k = head dim, n = query head of the group).
  uint32_t qf[NG][KS][2];
  {
    const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(pb.q);
#pragma unroll
    for (int nt = 0; nt < NG; ++nt) {
      const int g = nt * 8 + (lane >> 2);
      const bool ok = g < G;
      const uint32_t *qrow =
          reinterpret_cast<const uint32_t *>(q + ((size_t)it.token * pb.hq + hk * G + (ok ? g : 0)) * D);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qf[nt][ks][0] = ok ? qrow[ks * 8 + (lane & 3)] : 0u;
        qf[nt][ks][1] = ok ? qrow[ks * 8 + 4 + (lane & 3)] : 0u;
      }
    }
  }

  float o[KS][NG][4];
  float m_run[NG][2], l_run[NG][2];
#pragma unroll
  for (int nt = 0; nt < NG; ++nt) {
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
  }

  // per-lane ldmatrix geometry
  const int rk = (lane & 7) + ((lane >> 3) & 1) * 8;   // K: token row
  const int ck = lane >> 4;                            // K: chunk offset within a k-step
  const int rv = (lane & 7) + ((lane >> 4) & 1) * 8;   // V: token row
  const int cv = (lane >> 3) & 1;                      // V: chunk offset within an m-tile
  bool timed_out = false;
  bool touched = false;   // a stage was written through the generic proxy
  int k_stop = 0;         // first block index this warp did not consume

  for (int k = 0;; ++k) {
    k_stop = k;
    const int b = it.blk_begin + (PACK ? k : warp + kWarps * k);
    if (b >= it.blk_end) break;
    const int st = k % NST;
    if (!ptx::mbar_wait(&my_bars[st], (uint32_t)((k / NST) & 1))) {
      timed_out = true;
      break;
    }
    uint8_t *sk = my_ring + st * S::kStage;
    uint8_t *sv = sk + S::kHalves * S::kTile;

    // Rows without a loaded cache entry: the new token (from k_new / v_new,
    // also stored to its cache slot here), past-the-end rows and rows of
    // unreadable pages (zeros).
    bool bad = false;
    for (int r0 = 0; r0 < 16; r0 += box_rows) {
      const int pos = b * 16 + r0;
      if (pos < c && my_pages[pos / P - first_page] < 0) bad = true;
    }
    if (b == nblk_total - 1 || bad) {
      touched = true;
      const __nv_bfloat16 *kn = reinterpret_cast<const __nv_bfloat16 *>(pb.k_new);
      const __nv_bfloat16 *vn = reinterpret_cast<const __nv_bfloat16 *>(pb.v_new);
      __nv_bfloat16 *kc = reinterpret_cast<__nv_bfloat16 *>(pb.k_cache);
      __nv_bfloat16 *vc = reinterpret_cast<__nv_bfloat16 *>(pb.v_cache);
      for (int idx = lane; idx < 16 * (D / 8); idx += 32) {
        const int r = idx / (D / 8);
        const int ch = idx % (D / 8);
        const int pos = b * 16 + r;
        if (pos < c && my_pages[pos / P - first_page] >= 0) continue;
        uint4 kval = make_uint4(0, 0, 0, 0), vval = make_uint4(0, 0, 0, 0);
        if (pos == c) {
          const size_t src = ((size_t)it.token * pb.hkv + hk) * D + ch * 8;
          kval = *reinterpret_cast<const uint4 *>(kn + src);
          vval = *reinterpret_cast<const uint4 *>(vn + src);
          const int pg = my_pages[c / P - first_page];
          if (kCacheWrite && pg >= 0) {
            const size_t dst = (((size_t)pg * P + c % P) * pb.hkv + hk) * D + ch * 8;
            *reinterpret_cast<uint4 *>(kc + dst) = kval;
            *reinterpret_cast<uint4 *>(vc + dst) = vval;
          }
        }
        *reinterpret_cast<uint4 *>(sk + tile_off(r, ch)) = kval;
        *reinterpret_cast<uint4 *>(sv + tile_off(r, ch)) = vval;
      }
      __syncwarp();
    }

    // S^T = K Q^T  (16 tokens x 8 heads per n-tile)
    float s[NG][4];
#pragma unroll
    for (int nt = 0; nt < NG; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    const uint32_t sk_u = ptx::smem_u32(sk);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t a[4];
      ptx::ldmatrix_x4(a[0], a[1], a[2], a[3], sk_u + tile_off(rk, 2 * ks + ck));
#pragma unroll
      for (int nt = 0; nt < NG; ++nt) ptx::mma_bf16_16816(s[nt], a, qf[nt][ks][0], qf[nt][ks][1]);
    }

    // online softmax over this block, per query head (column)
    const bool v0 = b * 16 + (lane >> 2) < kv;
    const bool v1 = b * 16 + (lane >> 2) + 8 < kv;
    uint32_t pb0[NG], pb1[NG];
#pragma unroll
    for (int nt = 0; nt < NG; ++nt) {
      float x0 = v0 ? s[nt][0] * scale_log2 : -INFINITY;
      float x1 = v0 ? s[nt][1] * scale_log2 : -INFINITY;
      float x2 = v1 ? s[nt][2] * scale_log2 : -INFINITY;
      float x3 = v1 ? s[nt][3] * scale_log2 : -INFINITY;
      float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
      const float al0 = ptx::ex2(m_run[nt][0] - mn0), al1 = ptx::ex2(m_run[nt][1] - mn1);
      m_run[nt][0] = mn0;
      m_run[nt][1] = mn1;
      const float p0 = ptx::ex2(x0 - mn0), p1 = ptx::ex2(x1 - mn1);
      const float p2 = ptx::ex2(x2 - mn0), p3 = ptx::ex2(x3 - mn1);
      // l sums the fp32 weights: the max is updated every block, so the
      // largest weight is exactly 1 and the bf16 rounding of the others
      // moves O by far less than a bf16 step
      l_run[nt][0] = l_run[nt][0] * al0 + p0 + p2;
      l_run[nt][1] = l_run[nt][1] * al1 + p1 + p3;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        o[mt][nt][0] *= al0;
        o[mt][nt][1] *= al1;
        o[mt][nt][2] *= al0;
        o[mt][nt][3] *= al1;
      }
      pb0[nt] = ptx::movmatrix_trans(ptx::pack_bf16(p0, p1));
      pb1[nt] = ptx::movmatrix_trans(ptx::pack_bf16(p2, p3));
    }

    // O^T += V^T P^T
    const uint32_t sv_u = ptx::smem_u32(sv);
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
      uint32_t a[4];
      ptx::ldmatrix_x4_trans(a[0], a[1], a[2], a[3], sv_u + tile_off(rv, 2 * mt + cv));
#pragma unroll
      for (int nt = 0; nt < NG; ++nt) ptx::mma_bf16_16816(o[mt][nt], a, pb0[nt], pb1[nt]);
    }
    __syncwarp();
    if (lane == 0) {
      if (touched) ptx::fence_proxy_async_smem();
      issue(k + NST);
    }
  }

  if (timed_out && lane == 0) atomicOr(pb.err, RPA_DEV_TIMEOUT);
  // finish the row sums across the 8 lanes that share a column
#pragma unroll
  for (int nt = 0; nt < NG; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) l_run[nt][j] += __shfl_xor_sync(0xffffffffu, l_run[nt][j], off);

  // after a timeout, wait (bounded) for the copies this warp queued but did
  // not consume, so none lands after the CTA has gone
  if (timed_out && lane == 0) {
    for (int k = k_stop; k < k_stop + NST; ++k)
      if (it.blk_begin + (PACK ? k : warp + kWarps * k) < it.blk_end)
        ptx::mbar_wait(&my_bars[k % NST], (uint32_t)((k / NST) & 1));
  }

  if (PACK) {
    // this warp's item alone: out = O / l straight from the fragments (lane
    // holds head g0 = 8 nt + 2 (lane % 4) [+1], dims 16 mt + lane / 4 [+8])
    if (!has_item) return;
#pragma unroll
    for (int nt = 0; nt < NG; ++nt) {
      const int g0 = nt * 8 + 2 * (lane & 3);
      // head g0 + j takes o[.][nt][j] (dim d0) and o[.][nt][j + 2] (dim d0 + 8)
      float ov[2][KS][2];
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        ov[0][mt][0] = o[mt][nt][0];
        ov[0][mt][1] = o[mt][nt][2];
        ov[1][mt][0] = o[mt][nt][1];
        ov[1][mt][1] = o[mt][nt][3];
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int g = g0 + j;
        if (g < G) {
          const float inv = 1.f / l_run[nt][j];
          const float lse = (m_run[nt][j] + log2f(l_run[nt][j])) * kLn2;
          const int h = hk * G + g;
#pragma unroll
          for (int mt = 0; mt < KS; ++mt) {
            const int d0 = mt * 16 + (lane >> 2);
            const float v0 = ov[j][mt][0] * inv, v1 = ov[j][mt][1] * inv;
            if (it.partial < 0) {
              __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(pb.out) + ((size_t)it.token * pb.hq + h) * D;
              out[d0] = __float2bfloat16_rn(v0);
              out[d0 + 8] = __float2bfloat16_rn(v1);
            } else {
              const size_t row = ((size_t)it.partial * pb.hkv + hk) * G + g;
              part_o[row * D + d0] = v0;
              part_o[row * D + d0 + 8] = v1;
            }
          }
          if ((lane >> 2) == 0) {
            if (it.partial < 0) {
              if (pb.lse != nullptr) pb.lse[(size_t)it.token * pb.hq + h] = lse;
            } else {
              part_lse[((size_t)it.partial * pb.hkv + hk) * G + g] = lse;
            }
          }
        }
      }
    }
    return;
  }
  __syncthreads();

  // merge the four warps' partial softmax states through shared memory
  float *mo = reinterpret_cast<float *>(ring);            // [warp][g][D]
  float *mm = mo + kWarps * 16 * D;                        // [warp][16]
  float *ml = mm + kWarps * 16;                            // [warp][16]
#pragma unroll
  for (int nt = 0; nt < NG; ++nt) {
    const int g0 = nt * 8 + 2 * (lane & 3);
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
      const int d0 = mt * 16 + (lane >> 2);
      if (g0 < G) {
        mo[(warp * 16 + g0) * D + d0] = o[mt][nt][0];
        mo[(warp * 16 + g0) * D + d0 + 8] = o[mt][nt][2];
      }
      if (g0 + 1 < G) {
        mo[(warp * 16 + g0 + 1) * D + d0] = o[mt][nt][1];
        mo[(warp * 16 + g0 + 1) * D + d0 + 8] = o[mt][nt][3];
      }
    }
    if (lane < 4) {
      mm[warp * 16 + g0] = m_run[nt][0];
      mm[warp * 16 + g0 + 1] = m_run[nt][1];
      ml[warp * 16 + g0] = l_run[nt][0];
      ml[warp * 16 + g0 + 1] = l_run[nt][1];
    }
  }
  __syncthreads();

  for (int idx = tid; idx < G * D; idx += blockDim.x) {
    const int g = idx / D;
    const int d = idx % D;
    float mstar = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mstar = fmaxf(mstar, mm[w * 16 + g]);
    float acc = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float wt = ptx::ex2(mm[w * 16 + g] - mstar);   // 0 for a warp with no blocks
      acc += wt * mo[(w * 16 + g) * D + d];
      lsum += wt * ml[w * 16 + g];
    }
    const float val = acc / lsum;
    const float lse = (mstar + log2f(lsum)) * kLn2;
    if (it.partial < 0) {
      __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(pb.out);
      out[((size_t)it.token * pb.hq + hk * G + g) * D + d] = __float2bfloat16_rn(val);
      if (d == 0 && pb.lse != nullptr) pb.lse[(size_t)it.token * pb.hq + hk * G + g] = lse;
    } else {
      const size_t row = ((size_t)it.partial * pb.hkv + hk) * G + g;
      part_o[row * D + d] = val;
      if (d == 0) part_lse[row] = lse;
    }
  }
}

template <int D, int NG, bool PACK>
__global__ void __launch_bounds__(128) decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                     const __grid_constant__ CUtensorMap tm_v,
                                                     const Problem pb, const DecodeItem *__restrict__ items,
                                                     int n_items, float *__restrict__ part_o,
                                                     float *__restrict__ part_lse, float scale_log2) {
  decode_body<D, NG, PACK>(tm_k, tm_v, pb, items, n_items, part_o, part_lse, scale_log2);
}

// The work items of a small host-planned decode batch, passed by value in the
// launch itself, so that no plan copy has to reach the device first.
constexpr int kInlineItems = 900;    // 28.8 KB of kernel parameters
struct DecodeInline {
  DecodeItem items[kInlineItems];
};

template <int D, int NG>
__global__ void __launch_bounds__(128) decode_inline_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                            const __grid_constant__ CUtensorMap tm_v,
                                                            const Problem pb, const __grid_constant__ DecodeInline plan,
                                                            int n_items, float *__restrict__ part_o,
                                                            float *__restrict__ part_lse, float scale_log2) {
  decode_body<D, NG, false>(tm_k, tm_v, pb, plan.items, n_items, part_o, part_lse, scale_log2);
}

// One warp per (sequence, query head): merge the normalised partial outputs
// of the sequence's chunks with weights exp(lse_i - lse), lse = log sum exp.
template <int D>
__device__ __forceinline__ void combine_body(const Problem &pb, const CombineItem *__restrict__ items,
                                             int n_items, const float *__restrict__ part_o,
                                             const float *__restrict__ part_lse) {
  constexpr int E = D / 32;
  // launched right behind the decode grid (programmatic dependent launch):
  // its partial results are complete and visible after this wait
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (pb.dev_counts != nullptr) n_items = min(n_items, pb.dev_counts[kCntCombine]);
  if (w >= (long long)n_items * pb.hq) return;
  const CombineItem ci = items[w / pb.hq];
  const int h = (int)(w % pb.hq);
  const int G = pb.hq / pb.hkv;
  const int hk = h / G, g = h % G;
  float mstar = -INFINITY;
  for (int j = lane; j < ci.nsplit; j += 32)
    mstar = fmaxf(mstar, part_lse[((size_t)(ci.first_partial + j) * pb.hkv + hk) * G + g]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mstar = fmaxf(mstar, __shfl_xor_sync(0xffffffffu, mstar, off));
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float wsum = 0.f;
  for (int j = 0; j < ci.nsplit; ++j) {
    const size_t row = ((size_t)(ci.first_partial + j) * pb.hkv + hk) * G + g;
    const float wt = __expf(part_lse[row] - mstar);
    wsum += wt;
    const float *src = part_o + row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 4) {
      const float4 v = *reinterpret_cast<const float4 *>(src + e);
      acc[e] += wt * v.x;
      acc[e + 1] += wt * v.y;
      acc[e + 2] += wt * v.z;
      acc[e + 3] += wt * v.w;
    }
  }
  __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(pb.out) + ((size_t)ci.token * pb.hq + h) * D + lane * E;
  const float inv = 1.f / wsum;
#pragma unroll
  for (int e = 0; e < E; ++e) out[e] = __float2bfloat16_rn(acc[e] * inv);
  if (lane == 0 && pb.lse != nullptr) pb.lse[(size_t)ci.token * pb.hq + h] = mstar + logf(wsum);
}

template <int D>
__global__ void __launch_bounds__(128) combine_kernel(const Problem pb, const CombineItem *__restrict__ items,
                                                      int n_items, const float *__restrict__ part_o,
                                                      const float *__restrict__ part_lse) {
  combine_body<D>(pb, items, n_items, part_o, part_lse);
}

constexpr int kInlineRows = 1800;   // 28.8 KB of kernel parameters
struct CombineInline {
  CombineItem rows[kInlineRows];
};

template <int D>
__global__ void __launch_bounds__(128) combine_inline_kernel(const Problem pb, const __grid_constant__ CombineInline plan,
                                                             int n_items, const float *__restrict__ part_o,
                                                             const float *__restrict__ part_lse) {
  combine_body<D>(pb, plan.rows, n_items, part_o, part_lse);
}

bool decode_maps(const Problem &pb, int D, CUtensorMap *tk, CUtensorMap *tv) {
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)pb.hkv, (uint64_t)pb.num_pages * pb.p};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)pb.hkv * D * 2};
  const uint32_t box[3] = {64, 1, (uint32_t)(pb.p < 16 ? pb.p : 16)};
  return make_tmap_bf16_3d(tk, pb.k_cache, dims, strides, box, true) &&
         make_tmap_bf16_3d(tv, pb.v_cache, dims, strides, box, true);
}

template <int D, int NG, bool PACK>
cudaError_t launch_decode_t(const Problem &pb, const DecodeItem *items, int n_items, float *po, float *pl,
                            cudaStream_t stream) {
  using S = DecodeShape<D>;
  CUtensorMap tk, tv;
  if (!decode_maps(pb, D, &tk, &tv)) return cudaErrorInvalidValue;
  auto kern = decode_kernel<D, NG, PACK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(PACK ? (n_items + kWarps - 1) / kWarps : n_items), (unsigned)pb.hkv);
  kern<<<grid, kWarps * 32, S::kSmem, stream>>>(tk, tv, pb, items, n_items, po, pl, pb.scale * kLog2e);
  return cudaGetLastError();
}

template <int D, int NG>
cudaError_t launch_decode_inline_t(const Problem &pb, const DecodeItem *host_items, int n_items, float *po,
                                   float *pl, cudaStream_t stream) {
  using S = DecodeShape<D>;
  CUtensorMap tk, tv;
  if (!decode_maps(pb, D, &tk, &tv)) return cudaErrorInvalidValue;
  auto kern = decode_inline_kernel<D, NG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem);
  if (e != cudaSuccess) return e;
  static thread_local DecodeInline plan;   // parameter staging (the launch copies it)
  memcpy(plan.items, host_items, (size_t)n_items * sizeof(DecodeItem));
  dim3 grid((unsigned)n_items, (unsigned)pb.hkv);
  kern<<<grid, kWarps * 32, S::kSmem, stream>>>(tk, tv, pb, plan, n_items, po, pl, pb.scale * kLog2e);
  return cudaGetLastError();
}

// The combine queued right behind the decode grid with programmatic
// dependent launch (when `pdl`): its CTAs may start during the decode tail
// and wait on the device for the decode results.
template <typename K, typename... Args>
cudaError_t launch_combine_grid(K kern, unsigned blocks, bool pdl, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(blocks, 1, 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  if (pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const Problem &pb, const DecodeItem *items, int n_items, float *partial_o,
                          float *partial_lse, bool pack, cudaStream_t stream) {
  if (n_items <= 0) return cudaSuccess;
  const int G = pb.hq / pb.hkv;
  const bool two = G > 8;
#define RPA_DECODE_CASE(DD)                                                                              \
  case DD:                                                                                               \
    if (pack)                                                                                            \
      return two ? launch_decode_t<DD, 2, true>(pb, items, n_items, partial_o, partial_lse, stream)      \
                 : launch_decode_t<DD, 1, true>(pb, items, n_items, partial_o, partial_lse, stream);     \
    return two ? launch_decode_t<DD, 2, false>(pb, items, n_items, partial_o, partial_lse, stream)       \
               : launch_decode_t<DD, 1, false>(pb, items, n_items, partial_o, partial_lse, stream);
  switch (pb.d) {
    RPA_DECODE_CASE(64)
    RPA_DECODE_CASE(128)
    RPA_DECODE_CASE(256)
    default: return cudaErrorInvalidValue;
  }
#undef RPA_DECODE_CASE
}

cudaError_t launch_combine(const Problem &pb, const CombineItem *items, int n_items, const float *partial_o,
                           const float *partial_lse, cudaStream_t stream, bool pdl) {
  if (n_items <= 0) return cudaSuccess;
  const long long warps = (long long)n_items * pb.hq;
  const unsigned blocks = (unsigned)((warps + 3) / 4);
  switch (pb.d) {
    case 64: return launch_combine_grid(combine_kernel<64>, blocks, pdl, stream, pb, items, n_items, partial_o, partial_lse);
    case 128: return launch_combine_grid(combine_kernel<128>, blocks, pdl, stream, pb, items, n_items, partial_o, partial_lse);
    case 256: return launch_combine_grid(combine_kernel<256>, blocks, pdl, stream, pb, items, n_items, partial_o, partial_lse);
    default: return cudaErrorInvalidValue;
  }
}

bool decode_plan_fits_inline(int n_items, int n_combine) {
  return n_items <= kInlineItems && n_combine <= kInlineRows;
}

cudaError_t launch_decode_inline(const Problem &pb, const DecodeItem *host_items, int n_items, float *partial_o,
                                 float *partial_lse, cudaStream_t stream) {
  if (n_items <= 0) return cudaSuccess;
  if (n_items > kInlineItems) return cudaErrorInvalidValue;
  const bool two = pb.hq / pb.hkv > 8;
  switch (pb.d) {
    case 64: return two ? launch_decode_inline_t<64, 2>(pb, host_items, n_items, partial_o, partial_lse, stream)
                        : launch_decode_inline_t<64, 1>(pb, host_items, n_items, partial_o, partial_lse, stream);
    case 128: return two ? launch_decode_inline_t<128, 2>(pb, host_items, n_items, partial_o, partial_lse, stream)
                         : launch_decode_inline_t<128, 1>(pb, host_items, n_items, partial_o, partial_lse, stream);
    case 256: return two ? launch_decode_inline_t<256, 2>(pb, host_items, n_items, partial_o, partial_lse, stream)
                         : launch_decode_inline_t<256, 1>(pb, host_items, n_items, partial_o, partial_lse, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_combine_inline(const Problem &pb, const CombineItem *host_rows, int n_items,
                                  const float *partial_o, const float *partial_lse, cudaStream_t stream, bool pdl) {
  if (n_items <= 0) return cudaSuccess;
  if (n_items > kInlineRows) return cudaErrorInvalidValue;
  static thread_local CombineInline plan;   // parameter staging (the launch copies it)
  memcpy(plan.rows, host_rows, (size_t)n_items * sizeof(CombineItem));
  const long long warps = (long long)n_items * pb.hq;
  const unsigned blocks = (unsigned)((warps + 3) / 4);
  switch (pb.d) {
    case 64: return launch_combine_grid(combine_inline_kernel<64>, blocks, pdl, stream, pb, plan, n_items, partial_o, partial_lse);
    case 128: return launch_combine_grid(combine_inline_kernel<128>, blocks, pdl, stream, pb, plan, n_items, partial_o, partial_lse);
    case 256: return launch_combine_grid(combine_inline_kernel<256>, blocks, pdl, stream, pb, plan, n_items, partial_o, partial_lse);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rpa
