// prefill_kernel.cu -- prefill and chunked-prefill attention on the 5th
// generation tensor cores (tcgen05 + TMEM), with the fused cache update.
//
// The pages measure prefill against the matrix units' peak (talk summary,
// 00:11:09: up to 73 % MFU, 63 % with a causal mask) and fuse the KV-cache
// write into the attention kernel (00:06:36).  On B200 one CTA computes one
// 128-row tile of new tokens for one query head:
//
//   warps 0-3  softmax: one query row per thread; S rows come out of TMEM
//              (tcgen05.ld), P goes back into TMEM as bf16 (tcgen05.st),
//              online softmax in log2 units with a lazily refreshed running
//              max (O is rescaled only when the max grows by more than 2^8);
//              epilogue O / l -> bf16, lse.  Before the first block (while
//              Q and the first S are on their way) they copy the tile's
//              share of the new K/V rows into its cache pages.
//   warp 4     producer: TMA of the Q tile, then K and V blocks of BN keys
//              into rings of their own (K as soon as its stage is free):
//              cached context from the pages (one box per page segment),
//              new tokens from k_new / v_new.  Rows of a block that hold no
//              valid key (past the context, past the sequence, bad pages)
//              are zeroed before the block is released, so stale or NaN
//              slots never reach the tensor cores.
//   warp 5     TMEM owner and MMA issue (all lanes run the loop, one elected
//              lane issues): S = Q K^T into one of two TMEM buffers, then
//              O += P V with P read from TMEM.  The producer warp issues its
//              copies the same way.
//
// Keys are ordered as context blocks [0, c) followed by new-token blocks
// starting at c, so with BN = 128 the causal diagonal of a 128-row tile is
// exactly one block.
//
// At head_dim 256 this kernel is selectable (RPA_OPT_PREFILL_KERNEL = 1); the
// default there is the CTA-pair kernel of prefill3_kernel.cu, whose MMAs
// outpace this one-tile-per-CTA design.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "kernels.h"
#include "ptx.cuh"
#include "tma.h"

namespace rpa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

template <int D>
struct PrefillShape {
  static constexpr int BM = kPrefillTileRows;          // 128 query rows
  static constexpr int BN = D == 256 ? 64 : 128;       // keys per block
  // K and V rings of their own: a block's K is needed first (QK(j) comes
  // before PV(j-1)), its V a softmax later
  static constexpr int NSK = 3;                        // K stages
  static constexpr int NSV = 2;                        // V stages
  static constexpr int kHalves = D / 64;
  static constexpr int kQBytes = kHalves * BM * 128;
  static constexpr int kKVBytes = kHalves * BN * 128;  // one K or one V block
  static constexpr int kData = kQBytes + (NSK + NSV) * kKVBytes;
  static constexpr int kBarriers = 32;
  // at least 116 KB so that two CTAs never share an SM (each owns all 512
  // TMEM columns)
  static constexpr int kSmemUsed = 1024 + kData + kBarriers * 8 + 64;
  static constexpr int kSmem = kSmemUsed > 116 * 1024 ? kSmemUsed : 116 * 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = BN, kColO = 2 * BN;
  static_assert(kColO + D <= kTmemCols, "TMEM budget");
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[3], k_empty[3], v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t fix, drain;
};

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         uint32_t *err) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (ptx::globaltimer() - t0 > ptx::kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(err, RPA_DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// wait_bar by every lane of a warp, with a warp-uniform result.
__device__ __forceinline__ bool wait_all1(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint32_t *err) {
  return __all_sync(0xffffffffu, wait_bar(bar, parity, abort_flag, err));
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                   const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kn,
                   const __grid_constant__ CUtensorMap tm_vn, const Problem pb,
                   const PrefillTile *__restrict__ tiles, float scale_log2) {
  using S = PrefillShape<D>;
  constexpr int BM = S::BM, BN = S::BN, NSK = S::NSK, NSV = S::NSV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = base;
  uint8_t *sK = sQ + S::kQBytes;                 // NSK blocks
  uint8_t *sV = sK + NSK * S::kKVBytes;          // NSV blocks
  Bars *bars = reinterpret_cast<Bars *>(base + S::kData);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  // capacity-sized grid of a device-planned call: CTAs past the tiles leave
  if (pb.dev_counts != nullptr && (int)blockIdx.y >= pb.dev_counts[kCntPrefill]) return;
  const PrefillTile tile = tiles[blockIdx.y];
  const int h = blockIdx.x;
  const int G = pb.hq / pb.hkv;
  const int hk = h / G;
  const int c = tile.kv_len - tile.q_len;             // cached context length
  const int r0 = tile.tile_row;
  const int n_ctx = (c + BN - 1) / BN;
  const int n_new = pb.causal ? (r0 + tile.rows + BN - 1) / BN : (tile.q_len + BN - 1) / BN;
  const int nb = n_ctx + n_new;
  const int32_t *pt_row = pb.page_table + (size_t)tile.seq * pb.max_pages;

  if (tid == 0) {
    ptx::mbar_init(&bars->q_full, 1);
    for (int i = 0; i < NSK; ++i) {
      ptx::mbar_init(&bars->k_full[i], 1);
      ptx::mbar_init(&bars->k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->v_full[i], 1);
      ptx::mbar_init(&bars->v_empty[i], 1);
      ptx::mbar_init(&bars->s_full[i], 1);
      ptx::mbar_init(&bars->p_full[i], 128);
      ptx::mbar_init(&bars->pv_done[i], 1);
    }
    ptx::mbar_init(&bars->fix, 1);
    ptx::mbar_init(&bars->drain, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 5) {
    ptx::tmem_alloc(tmem_slot, S::kTmemCols);
    ptx::tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    ptx::tma_prefetch_desc(&tm_q);
    ptx::tma_prefetch_desc(&tm_kc);
    ptx::tma_prefetch_desc(&tm_vc);
    ptx::tma_prefetch_desc(&tm_kn);
    ptx::tma_prefetch_desc(&tm_vn);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    const int br = pb.p < BN ? pb.p : BN;      // rows per page-segment box
    const int nseg = BN / br;                  // <= 16
    uint32_t fix_phase = 0;
    int gk = 0, gv = 0;                        // blocks whose K (V) copies were queued and published
    bool fix_pending = false;
    ptx::mbar_arrive_expect_tx_elect(&bars->q_full, S::kQBytes);
    // Q is read once: first out of L2, ahead of the K/V blocks that the
    // other query heads and later tiles of the sequence read again
    const uint64_t once = ptx::l2_evict_first_policy();
    for (int hh = 0; hh < S::kHalves; ++hh)
      ptx::tma_load_3d_hint_elect(sQ + hh * BM * 128, &tm_q, &bars->q_full, hh * 64, h, tile.q_start + r0, once);
    for (int j = 0; j < nb; ++j) {
      const int sk = j % NSK, sv = j % NSV;
      const uint32_t phk = (uint32_t)((j / NSK) & 1), phv = (uint32_t)((j / NSV) & 1);
      uint8_t *dk = sK + sk * S::kKVBytes;
      uint8_t *dv = sV + sv * S::kKVBytes;
      // Block geometry: valid rows; for context blocks the page of each
      // segment (lane sg reads segment sg's page-table entry).
      const bool ctx = j < n_ctx;
      const int pos0 = ctx ? j * BN : (j - n_ctx) * BN;   // first position / new-token index
      const int valid = min(BN, (ctx ? c : tile.q_len) - pos0);
      int page = -1;
      bool seg_loaded = false, seg_bad = false;
      if (ctx && lane < nseg) {
        const int sp = pos0 + lane * br;
        if (sp < c) {
          page = pt_row[sp / pb.p];
          if (page < 0 || page >= pb.num_pages) {
            seg_bad = true;
            atomicOr(pb.err, RPA_DEV_BAD_PAGE);
          } else {
            seg_loaded = true;
          }
        }
      }
      const unsigned loaded_mask = __ballot_sync(0xffffffffu, seg_loaded);
      const bool fix = valid < BN || __any_sync(0xffffffffu, seg_bad);
      const uint32_t seg_bytes = (uint32_t)(S::kHalves * br * 128);
      const uint32_t blk_bytes = ctx ? (uint32_t)__popc(loaded_mask) * seg_bytes : (uint32_t)S::kKVBytes;

      // the copies of one operand (K or V) of this block into dst
      auto load = [&](uint8_t *dst, const CUtensorMap *tm_new, const CUtensorMap *tm_ctx, uint64_t *bar) {
        if (!ctx) {
          const int row = tile.q_start + pos0;
          for (int hh = 0; hh < S::kHalves; ++hh)
            ptx::tma_load_3d_elect(dst + hh * BN * 128, tm_new, bar, hh * 64, hk, row);
        } else {
          // each lane queues the copies of its own page segment, so one
          // instruction covers every segment of the block
          if ((loaded_mask >> lane) & 1u) {
            const int row = page * pb.p + ((pos0 + lane * br) % pb.p);
            for (int hh = 0; hh < S::kHalves; ++hh)
              ptx::tma_load_3d(dst + hh * BN * 128 + lane * br * 128, tm_ctx, bar, hh * 64, hk, row);
          }
          __syncwarp();
        }
      };
      if (!fix) {
        // K as soon as its stage is free, then V
        if (j >= NSK && !wait_all1(&bars->k_empty[sk], phk ^ 1u, abort_flag, pb.err)) break;
        ptx::mbar_arrive_expect_tx_elect(&bars->k_full[sk], blk_bytes);
        load(dk, &tm_kn, &tm_kc, &bars->k_full[sk]);
        ++gk;
        if (j >= NSV && !wait_all1(&bars->v_empty[sv], phv ^ 1u, abort_flag, pb.err)) break;
        ptx::mbar_arrive_expect_tx_elect(&bars->v_full[sv], blk_bytes);
        load(dv, &tm_vn, &tm_vc, &bars->v_full[sv]);
        ++gv;
        continue;
      }
      // Partial block or bad pages: both operands through the private
      // barrier (it completes even with no copies: the arrival carried zero
      // expected bytes), zero every row that holds no valid key, publish.
      if ((j >= NSK && !wait_all1(&bars->k_empty[sk], phk ^ 1u, abort_flag, pb.err)) ||
          (j >= NSV && !wait_all1(&bars->v_empty[sv], phv ^ 1u, abort_flag, pb.err)))
        break;
      ptx::mbar_arrive_expect_tx_elect(&bars->fix, 2 * blk_bytes);
      load(dk, &tm_kn, &tm_kc, &bars->fix);
      load(dv, &tm_vn, &tm_vc, &bars->fix);
      const bool fok = wait_all1(&bars->fix, fix_phase, abort_flag, pb.err);
      fix_phase ^= 1u;
      if (!fok) {
        fix_pending = true;   // copies may still be in flight: drained below
        break;
      }
      for (int r = lane; r < BN; r += 32) {
        const bool bad_row = r >= valid || (ctx && !((loaded_mask >> (r / br)) & 1u));
        if (!bad_row) continue;
        for (int hh = 0; hh < S::kHalves; ++hh) {
          uint4 *pk = reinterpret_cast<uint4 *>(dk + hh * BN * 128 + r * 128);
          uint4 *pv = reinterpret_cast<uint4 *>(dv + hh * BN * 128 + r * 128);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            pk[q] = make_uint4(0, 0, 0, 0);
            pv[q] = make_uint4(0, 0, 0, 0);
          }
        }
      }
      ptx::fence_proxy_async_smem();
      __syncwarp();
      ptx::mbar_arrive_elect(&bars->k_full[sk]);
      ptx::mbar_arrive_elect(&bars->v_full[sv]);
      ++gk;
      ++gv;
    }
    // Before the CTA can end, every copy this warp queued must have landed
    // (bounded waits; they complete without any other warp).
    if (lane == 0) {
      ptx::mbar_wait(&bars->q_full, 0);
      for (int j = gk - NSK < 0 ? 0 : gk - NSK; j < gk; ++j)
        ptx::mbar_wait(&bars->k_full[j % NSK], (uint32_t)((j / NSK) & 1));
      for (int j = gv - NSV < 0 ? 0 : gv - NSV; j < gv; ++j)
        ptx::mbar_wait(&bars->v_full[j % NSV], (uint32_t)((j / NSV) & 1));
      if (fix_pending) ptx::mbar_wait(&bars->fix, fix_phase ^ 1u);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA
    // All 32 lanes run the loop; one elected lane issues each MMA / commit.
    {
      const uint32_t tS0 = tmem + S::kColS0, tS1 = tmem + S::kColS1;
      const uint32_t tO = tmem + S::kColO;
      constexpr uint32_t idesc_qk = ptx::umma_idesc_bf16(128, BN, false);
      constexpr uint32_t idesc_pv = ptx::umma_idesc_bf16(128, D, true);
      const uint64_t dq0 = ptx::umma_desc_sw128(ptx::smem_u32(sQ), 16, 1024);
      const uint64_t dk0 = ptx::umma_desc_sw128(ptx::smem_u32(sK), 16, 1024);
      const uint64_t dv0 = ptx::umma_desc_sw128(ptx::smem_u32(sV), BN * 128, 1024);
      bool ok = wait_all1(&bars->q_full, 0, abort_flag, pb.err);
      auto pv = [&](int i) -> bool {
        const int b = i & 1, s = i % NSV;
        if (!wait_all1(&bars->p_full[b], (uint32_t)((i >> 1) & 1), abort_flag, pb.err)) return false;
        if (!wait_all1(&bars->v_full[s], (uint32_t)((i / NSV) & 1), abort_flag, pb.err)) return false;
        ptx::tc_fence_after();
        const uint64_t dv = dv0 + (uint64_t)((s * S::kKVBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          ptx::umma_ts_elect(tO, (b ? tS1 : tS0) + kk * 8, dv + (uint64_t)((kk * 16 * 128) >> 4), idesc_pv,
                             (i > 0 || kk > 0) ? 1u : 0u);
        ptx::umma_commit_elect(&bars->pv_done[b]);
        ptx::umma_commit_elect(&bars->v_empty[s]);
        return true;
      };
      // QK(j) writes the S buffer that PV(j-2) reads P from; it is issued
      // after PV(j-2) without waiting for it to finish, because tcgen05.mma
      // operations issued by one thread execute in issue order.
      for (int j = 0; ok && j < nb; ++j) {
        const int b = j & 1, s = j % NSK;
        if (!wait_all1(&bars->k_full[s], (uint32_t)((j / NSK) & 1), abort_flag, pb.err)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint64_t dk = dk0 + (uint64_t)((s * S::kKVBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          // 16 bf16 = 32 bytes inside a 128-byte row; 64-column tiles apart
          const uint32_t offq = ((ks >> 2) * BM * 128 + (ks & 3) * 32) >> 4;
          const uint32_t offk = ((ks >> 2) * BN * 128 + (ks & 3) * 32) >> 4;
          ptx::umma_ss_elect(b ? tS1 : tS0, dq0 + offq, dk + offk, idesc_qk, ks > 0 ? 1u : 0u);
        }
        ptx::umma_commit_elect(&bars->s_full[b]);
        ptx::umma_commit_elect(&bars->k_empty[s]);
        if (j >= 1 && !pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok) pv(nb - 1);
      // drain: wait until every MMA of this CTA has completed
      ptx::umma_commit_elect(&bars->drain);
      ptx::mbar_wait(&bars->drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    const int row = tid;                           // 0..127 == TMEM lane
    const int rn = r0 + row;                       // new-token index of this row
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    // Fused cache update, first: the softmax warps would otherwise wait for
    // Q and the first S.  The G CTAs of this KV head split the tile's new
    // rows between them; each row's K and V are copied into its page slot.
    {
      const int g = h % G;
      const int ra = (g * tile.rows) / G, rb = ((g + 1) * tile.rows) / G;
      const int chunks = D / 8;   // 16-byte chunks per row
      const __nv_bfloat16 *kn = reinterpret_cast<const __nv_bfloat16 *>(pb.k_new);
      const __nv_bfloat16 *vn = reinterpret_cast<const __nv_bfloat16 *>(pb.v_new);
      __nv_bfloat16 *kc = reinterpret_cast<__nv_bfloat16 *>(pb.k_cache);
      __nv_bfloat16 *vc = reinterpret_cast<__nv_bfloat16 *>(pb.v_cache);
      // kBatch chunks per thread in flight: the loads (sources and page-table
      // entries) of a batch are issued before its stores
      constexpr int kBatch = 8;
      const int total = kCacheWrite ? (rb - ra) * chunks : 0;
      for (int base = tid; base < total; base += 128 * kBatch) {
        uint4 kq[kBatch], vq[kBatch];
        int pgq[kBatch];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
          const int idx = base + q * 128;
          if (idx < total) {
            const int i = r0 + ra + idx / chunks;   // new-token index
            const size_t src = ((size_t)(tile.q_start + i) * pb.hkv + hk) * D + (idx % chunks) * 8;
            kq[q] = *reinterpret_cast<const uint4 *>(kn + src);
            vq[q] = *reinterpret_cast<const uint4 *>(vn + src);
            pgq[q] = pt_row[(c + i) / pb.p];
          }
        }
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
          const int idx = base + q * 128;
          if (idx >= total) continue;
          const int i = r0 + ra + idx / chunks, ch = idx % chunks;
          const int pos = c + i;
          const int pg = pgq[q];
          if (pg < 0 || pg >= pb.num_pages) {
            if (ch == 0) atomicOr(pb.err, RPA_DEV_BAD_PAGE);
            continue;
          }
          const size_t dst = (((size_t)pg * pb.p + pos % pb.p) * pb.hkv + hk) * D + ch * 8;
          *reinterpret_cast<uint4 *>(kc + dst) = kq[q];
          *reinterpret_cast<uint4 *>(vc + dst) = vq[q];
        }
      }
    }
    float m = -INFINITY, l = 0.f, lr = 0.f;   // lr: the normaliser of O (below)
    bool ok = true;
    for (int j = 0; j < nb; ++j) {
      const int b = j & 1;
      // warp-uniform decisions only: the tcgen05 loads and stores below are
      // warp-collective
      if (!__all_sync(0xffffffffu, wait_bar(&bars->s_full[b], (uint32_t)((j >> 1) & 1), abort_flag, pb.err))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t tS = lane_base + (b ? S::kColS1 : S::kColS0);
      float x[BN];
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc)
        ptx::tmem_ld32(tS + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&x[cc * 32]));
      ptx::tmem_ld_wait();
      // visible keys of this row in this block: the first `lim` columns
      const bool ctx = j < n_ctx;
      int lim;
      if (ctx) {
        lim = min(BN, c - j * BN);
      } else {
        const int kn0 = (j - n_ctx) * BN;
        const int end = pb.causal ? min(tile.q_len, rn + 1) : tile.q_len;
        lim = max(0, min(BN, end - kn0));
      }
      if (__any_sync(0xffffffffu, lim < BN)) {
#pragma unroll
        for (int i = 0; i < BN; ++i) x[i] = i < lim ? x[i] : -INFINITY;
      }
      // row max of the raw scores (scale > 0): 4 chains of 3-input max
      float mq[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
      for (int i = 4; i < BN; i += 8) {
        mq[0] = ptx::fmax3(mq[0], x[i], x[i + 1]);
        mq[1] = ptx::fmax3(mq[1], x[i + 2], x[i + 3]);
        if (i + 4 < BN) {
          mq[2] = ptx::fmax3(mq[2], x[i + 4], x[i + 5]);
          mq[3] = ptx::fmax3(mq[3], x[i + 6], x[i + 7]);
        }
      }
      const float mraw = ptx::fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3]));
      const float mx = mraw * scale_log2;
      const float m_new = fmaxf(m, mx);
      const bool need = m == -INFINITY ? false : (m_new > m + kRescaleThreshold);
      float alpha = 1.f;
      if (__any_sync(0xffffffffu, need)) {
        // O must hold every earlier block before it is rescaled
        if (j >= 1 && !__all_sync(0xffffffffu, wait_bar(&bars->pv_done[(j - 1) & 1],
                                                          (uint32_t)(((j - 1) >> 1) & 1), abort_flag, pb.err))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        alpha = (m_new == m) ? 1.f : ptx::ex2(m - m_new);
        if (j >= 1) {
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t r[32];
            ptx::tmem_ld32(lane_base + S::kColO + cc * 32, r);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            ptx::tmem_st32(lane_base + S::kColO + cc * 32, r);
          }
          ptx::tmem_st_wait();
        }
        m = m_new;
      } else if (m == -INFINITY) {
        m = m_new;
      }
      const float neg_m = m == -INFINITY ? 0.f : -m;
      const uint64_t scale2 = ptx::f2_pack(scale_log2, scale_log2);
      const uint64_t negm2 = ptx::f2_pack(neg_m, neg_m);
      uint64_t sp2[4] = {0, 0, 0, 0};   // packed partial sums
#pragma unroll
      for (int cc = 0; cc < BN / 64; ++cc) {
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float a0, a1;
          ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(x[cc * 64 + 2 * i], x[cc * 64 + 2 * i + 1]), scale2, negm2), a0, a1);
          const uint64_t pp = ptx::f2_pack(ptx::ex2(a0), ptx::ex2(a1));
          sp2[i & 3] = ptx::f2_add(sp2[i & 3], pp);
          float p0, p1;
          ptx::f2_unpack(pp, p0, p1);
          r[i] = ptx::pack_bf16(p0, p1);
        }
        ptx::tmem_st32(tS + cc * 32, r);
      }
      float spf[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) ptx::f2_unpack(sp2[k], spf[2 * k], spf[2 * k + 1]);
      const float sum = ((spf[0] + spf[1]) + (spf[2] + spf[3])) + ((spf[4] + spf[5]) + (spf[6] + spf[7]));
      // The PV MMA takes P rounded to bf16.  Under the lazy rescale the
      // block's largest weight can be up to 2^8 (not exactly 1), and its
      // rounding (relative 2^-9) moves O by up to 2^-9 |V| when one key
      // dominates the row.  lr, the normaliser of O, therefore counts that
      // weight as rounded, so that its rounding cancels in O / lr; the
      // other weights keep the error of a kernel whose max weight is 1.
      // l keeps the exact fp32 sum, for lse.
      const float pmax = ptx::ex2(fmaf(mraw, scale_log2, neg_m));   // as the loop computed it
      ptx::tmem_st_wait();
      l = l * alpha + sum;
      lr = lr * alpha + (sum - (pmax - ptx::round_bf16(pmax)));
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->p_full[b]);
    }
    // epilogue: O / l
    if (ok && __all_sync(0xffffffffu, wait_bar(&bars->pv_done[(nb - 1) & 1], (uint32_t)(((nb - 1) >> 1) & 1),
                                                abort_flag, pb.err))) {
      ptx::tc_fence_after();
      const float inv = 1.f / lr;
      const bool store = row < tile.rows;
      const uint64_t once = ptx::l2_evict_first_policy();   // written once: first out of L2
      __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(pb.out) +
                           ((size_t)(tile.q_start + rn) * pb.hq + h) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        ptx::tmem_ld32(lane_base + S::kColO + cc * 32, r);
        ptx::tmem_ld_wait();
        if (store) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = ptx::pack_bf16(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
          uint4 *dst = reinterpret_cast<uint4 *>(out + cc * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            ptx::st_global_hint(dst + i, make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]), once);
        }
      }
      if (store && pb.lse != nullptr) pb.lse[(size_t)(tile.q_start + rn) * pb.hq + h] = (m + log2f(l)) * kLn2;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 5) ptx::tmem_dealloc(tmem, S::kTmemCols);
}

template <int D>
cudaError_t launch_prefill_t(const Problem &pb, const PrefillTile *tiles, int n_tiles, cudaStream_t stream) {
  using S = PrefillShape<D>;
  CUtensorMap tq, tkc, tvc, tkn, tvn;
  const uint64_t qdims[3] = {(uint64_t)D, (uint64_t)pb.hq, (uint64_t)pb.total_q};
  const uint64_t qstr[2] = {(uint64_t)D * 2, (uint64_t)pb.hq * D * 2};
  const uint32_t qbox[3] = {64, 1, (uint32_t)S::BM};
  const uint64_t cdims[3] = {(uint64_t)D, (uint64_t)pb.hkv, (uint64_t)pb.num_pages * pb.p};
  const uint64_t cstr[2] = {(uint64_t)D * 2, (uint64_t)pb.hkv * D * 2};
  const uint32_t cbox[3] = {64, 1, (uint32_t)(pb.p < S::BN ? pb.p : S::BN)};
  const uint64_t ndims[3] = {(uint64_t)D, (uint64_t)pb.hkv, (uint64_t)pb.total_q};
  const uint64_t nstr[2] = {(uint64_t)D * 2, (uint64_t)pb.hkv * D * 2};
  const uint32_t nbox[3] = {64, 1, (uint32_t)S::BN};
  if (!make_tmap_bf16_3d(&tq, pb.q, qdims, qstr, qbox, true) ||
      !make_tmap_bf16_3d(&tkc, pb.k_cache, cdims, cstr, cbox, true) ||
      !make_tmap_bf16_3d(&tvc, pb.v_cache, cdims, cstr, cbox, true) ||
      !make_tmap_bf16_3d(&tkn, pb.k_new, ndims, nstr, nbox, true) ||
      !make_tmap_bf16_3d(&tvn, pb.v_new, ndims, nstr, nbox, true))
    return cudaErrorInvalidValue;
  auto kern = prefill_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)pb.hq, (unsigned)n_tiles);
  kern<<<grid, 192, S::kSmem, stream>>>(tq, tkc, tvc, tkn, tvn, pb, tiles, pb.scale * kLog2e);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const Problem &pb, const PrefillTile *tiles, int n_tiles, cudaStream_t stream) {
  if (n_tiles <= 0) return cudaSuccess;
  switch (pb.d) {
    case 256: return launch_prefill_t<256>(pb, tiles, n_tiles, stream);   // 64 / 128: prefill2
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rpa
