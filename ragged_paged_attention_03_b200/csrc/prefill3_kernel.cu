// prefill3_kernel.cu -- prefill / chunked-prefill attention with score
// tiles computed ahead of the softmax: while the softmax warps turn S(j) into
// P(j), the tensor cores compute the next block's S = Q K^T and an earlier
// block's O += P V, so a block costs the larger of the softmax time and the
// MMA time instead of their sum (the compute-bound prefill regime of the RPA
// talk summary, 00:11:09; the cache update of 00:06:36 is fused here too).
// It is the default prefill kernel at head_dim 256, where the MMA work of a
// block (QK at N = 128 plus PV at N = 256) outweighs its softmax; at head_dim
// 128 it is selectable (the two-tile kernel in prefill2_kernel.cu is faster).
//
// Two builds of one kernel:
//  * PAIR = true: a cluster of two CTAs on two SMs works on one 256-row work
//    item; rank 0 (the leader) issues tcgen05.mma.cta_group::2 with M = 256.
//    Each CTA keeps its own 128 query rows (A operand, its TMEM lanes of S, P
//    and O) and loads only half of every K/V block: keys [64 r, 64 r + 64) of
//    K and head-dim columns [64 r, 64 r + 64) of V for rank r, the halves of
//    B that the pair MMA expects from each CTA.  Every MMA reads B once for
//    both CTAs, which halves the shared-memory and L2 traffic per SM and the
//    MMA instructions per FLOP.
//  * PAIR = false: one CTA per 128-row tile, tcgen05.mma.cta_group::1 with
//    M = 128 and whole K/V blocks.
//
// Roles of each CTA (512 threads at 128 registers each; every role fits
// without spills, so the register file is not repartitioned):
//   warps 0-7   softmax, one query row per thread in each warpgroup:
//               warpgroup 0 takes keys [0, 64) of every block, warpgroup 1
//               keys [64, 128); the two threads of a row agree on its max
//               through shared memory, each turns its half of S(b) into P(b)
//               (bf16, back into S(b)'s columns: the A operand of the PV MMA)
//               and keeps its share of the row sum
//   warps 8-11  epilogue: O / l of a finished unit from TMEM to `out`, lse;
//               while a unit computes, four fifths of its cache update
//   warp 12     TMA producer of Q tiles (two buffers) and K blocks of 128
//               keys (context from cache pages, new tokens from k_new; rows
//               without a valid key zeroed)
//   warp 13     TMEM allocation; MMA issue (the leader's, in a pair)
//   warp 14     TMA producer of V blocks (as for K): V(b) waits for the PV
//               that last read its stage (PV(b - 4) at head_dim 128), which
//               is queued NS - 1 blocks behind its QK, so a producer shared
//               with K would hold every K load back by as much
//   warp 15     fused cache update: a fifth of this CTA's share of each
//               unit's new K/V rows copied into their page slots
//
// TMEM (512 columns, the same columns in both CTAs of a pair):
//   head_dim 128: S(0) | S(1) | S(2) | O, 128 columns each (NS = 3);
//   head_dim 256: S(0) | S(1) | O, with O 256 columns wide (NS = 2).
//   Blocks cycle through the NS score buffers; O holds one unit at a time.
//
// The MMA warp issues, per block b (counted over all units of the CTA):
//   QK(b) into S(b mod NS), then PV(b - NS + 1) from P(b - NS + 1).  QK(b)
//   therefore waits for no softmax: the buffer it overwrites was last read by
//   PV(b - NS), issued before it, and tcgen05 operations issued by one thread
//   execute in order.  At NS = 3, while the softmax warps turn S(b) into P(b),
//   S(b + 1) is already computed and S(b + 2) is being computed.  The same
//   order means that when S(b) is complete, PV(b - NS) is too, which bounds
//   how far any barrier below can lag behind its waiter to one phase.  The
//   first PV of a unit waits for the epilogue to have read the previous
//   unit's O.
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
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O when the max grows by > 2^8

template <bool PAIR, int HEAD_DIM>
struct P3 {
  static constexpr int D = HEAD_DIM;
  static constexpr int BM = 128;                 // query rows per CTA
  static constexpr int BN = 128;                 // keys per block
  static constexpr int NCTA = PAIR ? 2 : 1;
  static constexpr int KH = BN / NCTA;           // keys of each K block this CTA holds
  static constexpr int VC = D / NCTA;            // head-dim columns of each V block this CTA holds
  static constexpr int VH = VC / 64;             // 128-byte column slabs of a V block
  static constexpr int kQBytes = BM * D * 2;     // 32 KB (head_dim 128) / 64 KB (256)
  static constexpr int kKBytes = KH * D * 2;
  static constexpr int kVBytes = BN * VC * 2;
  // head_dim 128: two Q buffers (the next unit's Q loads during this one)
  // and deep K/V rings; head_dim 256 (pairs only): one Q buffer and two
  // stages each of half-blocks, 192 KB in all
  static constexpr int NQ = D == 128 ? 2 : 1;
  static constexpr int NSK = D == 128 ? (PAIR ? 4 : 2) : 2;
  static constexpr int NSV = D == 128 ? (PAIR ? 4 : 2) : 2;
  static constexpr int kData = NQ * kQBytes + NSK * kKBytes + NSV * kVBytes;
  static constexpr int HK = BN / 2;               // keys of a block per softmax warpgroup
  // [unit parity][l of keys 0-63, l of keys 64-127, m, lr of keys 0-63, lr of keys 64-127][row]
  // (l: sums of the fp32 weights, for lse; lr: the normalisers of O)
  static constexpr int kStatFloats = 2 * 5 * BM;
  static constexpr int kRedFloats = 2 * 2 * BM;    // [exchange parity][warpgroup][row]: partial row maxima
  static constexpr int kSmem = 1024 + kData + (kStatFloats + kRedFloats) * 4 + 512;
  static constexpr uint32_t kTmemCols = 512;
  // TMEM: NS score buffers of 128 columns, then O (D columns): three score
  // buffers at head_dim 128, two at 256
  static constexpr int NS = D == 128 ? 3 : 2;
  static constexpr uint32_t kColO = NS * 128;
  static constexpr int kLag = NS - 1;             // PV(b - kLag) is issued after QK(b)
  static constexpr uint32_t kSoftmaxArrivals = 8 * NCTA;   // one elected lane per softmax warp, per CTA
  static constexpr uint32_t kEpilogueArrivals = 4 * NCTA;  // one per epilogue warp, per CTA
  static_assert(kColO + D <= kTmemCols, "TMEM columns");
  static_assert(kSmem <= 232448, "shared memory per CTA");
  static_assert(PAIR || D == 128, "head_dim 256 runs on CTA pairs only");
};

struct Bars3 {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[3];     // QK into S(i) complete (committed to both CTAs)
  uint64_t p_full[3];     // P in S(i) in every CTA (leader's barrier)
  uint64_t pv_done[2];    // PV of a block with this parity complete
  uint64_t o_full;        // last PV of a unit complete
  uint64_t o_free;        // epilogue of every CTA has read O (leader's)
  uint64_t st_full[2], st_free[2];   // row statistics softmax -> epilogue (local)
  uint64_t xch[4][2];     // partial row maxima of rows [32 w, 32 w + 32), by exchange parity (local)
  uint64_t kfix, vfix;    // private barriers of partial blocks (local)
  uint64_t drain, exit_bar;
};

// ------------------------------------------------------------- waiting
struct Sync {
  Bars3 *bars;
  volatile int *abort_flag;
  uint32_t peer_abort;     // shared::cluster address of the peer's abort flag (pairs)
  uint32_t *err;
};

template <bool PAIR>
__device__ __forceinline__ void raise_abort(const Sync &sy) {
  *sy.abort_flag = 1;
  if constexpr (PAIR) asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(sy.peer_abort), "r"(1) : "memory");
}

// Bounded wait by one thread: false on timeout (then RPA_DEV_TIMEOUT is set
// and both CTAs of a pair are told to stop) or when the kernel is stopping.
template <bool PAIR>
__device__ __forceinline__ bool wait3(const Sync &sy, uint64_t *bar, uint32_t parity) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (*sy.abort_flag) return false;
    if (ptx::globaltimer() - t0 > ptx::kWaitLimitNs) {
      atomicOr(sy.err, RPA_DEV_TIMEOUT);
      raise_abort<PAIR>(sy);
      return false;
    }
  }
  return true;
}

// wait3 by every lane of a warp, with a warp-uniform result.
template <bool PAIR>
__device__ __forceinline__ bool wait_all3(const Sync &sy, uint64_t *bar, uint32_t parity) {
  return __all_sync(0xffffffffu, wait3<PAIR>(sy, bar, parity));
}

// shared::cluster address of a barrier in the leader (rank 0) of the pair;
// this CTA's own barrier without a pair.
template <bool PAIR>
__device__ __forceinline__ uint32_t leader_bar(uint64_t *bar) {
  if constexpr (PAIR) return ptx::mapa_shared(bar, 0);
  return ptx::smem_u32(bar);
}

// One elected lane arrives for the whole warp (after __syncwarp) on `bar`:
// the leader's copy of it in a pair (possibly in the other CTA), this CTA's
// own otherwise.
template <bool PAIR>
__device__ __forceinline__ void warp_arrive_leader(uint64_t *bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) {
    if constexpr (PAIR)
      ptx::mbar_arrive_cluster(ptx::mapa_shared(bar, 0));
    else
      ptx::mbar_arrive(bar);
  }
  __syncwarp();
}


// ------------------------------------------------------------ schedule
// Units: PAIR -- (256-row item, query head), both CTAs of the pair on the
// same unit; single -- (128-row half of an item, query head).  Groups (a
// pair, or one CTA) walk the unit list in snake order: round k takes unit
// k * G + g on even rounds and k * G + (G - 1 - g) on odd ones, so that with
// items sorted heaviest first every group gets a similar share of the work.
template <bool PAIR>
__device__ __forceinline__ int group_id() { return PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x; }
template <bool PAIR>
__device__ __forceinline__ int n_groups() { return PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x; }
template <bool PAIR>
__device__ __forceinline__ int unit_of(int k) {
  const int G = n_groups<PAIR>(), g = group_id<PAIR>();
  return k * G + ((k & 1) ? G - 1 - g : g);
}

struct Unit3 {
  PrefillTile tile;     // the 256-row item
  int h, hk, c;         // query head, its KV head, cached context length
  int my_r0, my_rows;   // this CTA's first new-token row and its row count
  int n_ctx, nb;        // context blocks; key blocks of the unit (both CTAs)
  bool end, skip;       // past the last unit; nothing for this CTA to do
};

template <bool PAIR>
__device__ __forceinline__ Unit3 make_unit3(const PrefillTile *tiles, int u, int n_units, const Problem &pb,
                                            int rank) {
  using S = P3<PAIR, 128>;   // rows and keys per block do not depend on D
  Unit3 w{};
  w.end = u >= n_units;
  if (w.end) return w;
  const int per_item = PAIR ? pb.hq : 2 * pb.hq;
  w.tile = tiles[u / per_item];
  if (w.tile.rows == 0) {   // end of a device-planned tile list
    w.end = true;
    return w;
  }
  w.h = u % pb.hq;
  const int half = PAIR ? rank : (u / pb.hq) & 1;
  w.hk = w.h / (pb.hq / pb.hkv);
  w.c = w.tile.kv_len - w.tile.q_len;
  w.my_r0 = w.tile.tile_row + half * S::BM;
  w.my_rows = min(S::BM, max(0, w.tile.rows - half * S::BM));
  w.skip = !PAIR && w.my_rows == 0;
  w.n_ctx = (w.c + S::BN - 1) / S::BN;
  // the unit's rows: the whole item for a pair, this CTA's tile otherwise
  const int last_row = PAIR ? w.tile.tile_row + w.tile.rows : w.my_r0 + w.my_rows;
  const int new_end = pb.causal ? last_row : w.tile.q_len;
  w.nb = w.n_ctx + (new_end + S::BN - 1) / S::BN;
  return w;
}

// ---------------------------------------------------------------- MMA
template <bool PAIR, int D>
__device__ __forceinline__ void mma_qk(uint32_t tS, uint64_t dq, uint64_t dk) {
  using S = P3<PAIR, D>;
  constexpr uint32_t idesc = ptx::umma_idesc_bf16(PAIR ? 256 : 128, S::BN, false);
#pragma unroll
  for (int ks = 0; ks < S::D / 16; ++ks) {
    const uint32_t offq = ((ks >> 2) * S::BM * 128 + (ks & 3) * 32) >> 4;
    const uint32_t offk = ((ks >> 2) * S::KH * 128 + (ks & 3) * 32) >> 4;
    if constexpr (PAIR)
      ptx::umma_ss_pair_elect(tS, dq + offq, dk + offk, idesc, ks > 0 ? 1u : 0u);
    else
      ptx::umma_ss_elect(tS, dq + offq, dk + offk, idesc, ks > 0 ? 1u : 0u);
  }
}

template <bool PAIR, int D>
__device__ __forceinline__ void mma_pv(uint32_t tO, uint32_t tP, uint64_t dv, bool first) {
  using S = P3<PAIR, D>;
  constexpr uint32_t idesc = ptx::umma_idesc_bf16(PAIR ? 256 : 128, S::D, true);
#pragma unroll
  for (int kk = 0; kk < S::BN / 16; ++kk) {
    const uint64_t b = dv + (uint64_t)((kk * 16 * 128) >> 4);
    if constexpr (PAIR)
      ptx::umma_ts_pair_elect(tO, tP + kk * 8, b, idesc, (!first || kk > 0) ? 1u : 0u);
    else
      ptx::umma_ts_elect(tO, tP + kk * 8, b, idesc, (!first || kk > 0) ? 1u : 0u);
  }
}

template <bool PAIR>
__device__ __forceinline__ void commit(uint64_t *bar) {
  if constexpr (PAIR)
    ptx::umma_commit_pair_mc_elect(bar, (uint16_t)0x3);
  else
    ptx::umma_commit_elect(bar);
}

struct PendingPV {
  int gb;      // global block index of the P to consume
  int gu;      // unit counter of that unit
  bool first, last;
};

template <bool PAIR, int D>
__device__ __forceinline__ bool issue_pending_pv(const Sync &sy, const PendingPV &pv, uint32_t tmem, uint64_t dv0) {
  using S = P3<PAIR, D>;
  Bars3 *bars = sy.bars;
  const int sb = pv.gb % S::NS;
  if (!wait_all3<PAIR>(sy, &bars->p_full[sb], (uint32_t)((pv.gb / S::NS) & 1))) return false;
  const int vs = pv.gb % S::NSV;
  if (!wait_all3<PAIR>(sy, &bars->v_full[vs], (uint32_t)((pv.gb / S::NSV) & 1))) return false;
  // the unit's first PV overwrites O: the epilogue of the previous unit must
  // have read it
  if (pv.first && pv.gu >= 1 && !wait_all3<PAIR>(sy, &bars->o_free, (uint32_t)((pv.gu - 1) & 1))) return false;
  ptx::tc_fence_after();
  mma_pv<PAIR, D>(tmem + S::kColO, tmem + sb * 128, dv0 + (uint64_t)((vs * S::kVBytes) >> 4), pv.first);
  commit<PAIR>(&bars->v_empty[vs]);
  commit<PAIR>(&bars->pv_done[pv.gb & 1]);
  if (pv.last) commit<PAIR>(&bars->o_full);
  return true;
}

template <bool PAIR, int D>
__device__ __forceinline__ void mma_loop(const Sync &sy, const Problem &pb, const PrefillTile *tiles, int n_units,
                                         uint32_t tmem, uint32_t q_addr, uint32_t k_addr, uint32_t v_addr) {
  using S = P3<PAIR, D>;
  Bars3 *bars = sy.bars;
  const uint64_t dq0 = ptx::umma_desc_sw128(q_addr, 16, 1024);
  const uint64_t dk0 = ptx::umma_desc_sw128(k_addr, 16, 1024);
  const uint64_t dv0 = ptx::umma_desc_sw128(v_addr, S::BN * 128, 1024);
  int gb = 0, gu = 0;
  bool ok = true;
  int npend = 0;          // PVs queued behind the QKs (at most kLag: pa, then pbv)
  PendingPV pa{}, pbv{};
  for (int k = 0; ok; ++k) {
    const Unit3 w = make_unit3<PAIR>(tiles, unit_of<PAIR>(k), n_units, pb, 0);
    if (w.end) break;
    if (w.skip) continue;
    const int qb = gu % S::NQ;
    ok = wait_all3<PAIR>(sy, &bars->q_full[qb], (uint32_t)((gu / S::NQ) & 1));
    for (int j = 0; ok && j < w.nb; ++j, ++gb) {
      const int ks = gb % S::NSK;
      ok = wait_all3<PAIR>(sy, &bars->k_full[ks], (uint32_t)((gb / S::NSK) & 1));
      if (!ok) break;
      ptx::tc_fence_after();
      mma_qk<PAIR, D>(tmem + (gb % S::NS) * 128, dq0 + (uint64_t)((qb * S::kQBytes) >> 4),
                   dk0 + (uint64_t)((ks * S::kKBytes) >> 4));
      commit<PAIR>(&bars->k_empty[ks]);
      commit<PAIR>(&bars->s_full[gb % S::NS]);
      if (j + 1 == w.nb) commit<PAIR>(&bars->q_empty[qb]);
      // queue PV(gb); issue PV(gb - kLag) now
      const PendingPV cur{gb, gu, j == 0, j + 1 == w.nb};
      if (npend == S::kLag) {
        ok = issue_pending_pv<PAIR, D>(sy, pa, tmem, dv0);
        if (S::kLag == 2) {
          pa = pbv;
          pbv = cur;
        } else {
          pa = cur;
        }
      } else if (npend == 1) {
        pbv = cur;
        npend = 2;
      } else {
        pa = cur;
        npend = 1;
      }
    }
    ++gu;
  }
  if (ok && npend >= 1) ok = issue_pending_pv<PAIR, D>(sy, pa, tmem, dv0);
  if (ok && npend == 2) issue_pending_pv<PAIR, D>(sy, pbv, tmem, dv0);
}

// ------------------------------------------------------------ producer
// One K or V block of this CTA: `rows` rows of `slabs` 128-byte column slabs
// (slab stride rows * 128 bytes), keys [key0, key0 + rows) of the block's
// source (cache pages for a context block, k_new / v_new rows otherwise),
// head-dim columns starting at col0.  A block whose rows are all valid and
// readable goes straight to `full`; otherwise it lands on the private
// barrier `fix`, rows without a valid key are zeroed, then `full` is told.
template <bool PAIR>
struct BlockLoad {
  uint8_t *dst;
  int rows, slabs, col0;
  const CUtensorMap *tm_ctx, *tm_new;
  int seg_rows;   // rows per page segment (context blocks)
};

template <bool PAIR>
__device__ __forceinline__ bool load_block(const Sync &sy, const Problem &pb, const Unit3 &w, const int32_t *pt_row,
                                           const BlockLoad<PAIR> &L, bool ctx, int key0, uint64_t *full,
                                           uint64_t *fix, uint32_t &fix_phase, bool &fix_pending) {
  const int lane = threadIdx.x & 31;
  const int limit = ctx ? w.c : w.tile.q_len;              // keys of the source
  const int valid = max(0, min(L.rows, limit - key0));     // leading valid rows
  const int nseg = L.rows / L.seg_rows;
  bool seg_loaded = false, seg_bad = false;
  int page = -1;
  if (ctx && lane < nseg && key0 + lane * L.seg_rows < w.c) {
    page = pt_row[(key0 + lane * L.seg_rows) / pb.p];
    if (page < 0 || page >= pb.num_pages) {
      seg_bad = true;
      atomicOr(pb.err, RPA_DEV_BAD_PAGE);
    } else {
      seg_loaded = true;
    }
  }
  const unsigned loaded = __ballot_sync(0xffffffffu, seg_loaded);
  const bool need_fix = valid < L.rows || __any_sync(0xffffffffu, seg_bad);
  const uint32_t seg_bytes = (uint32_t)(L.slabs * L.seg_rows * 128);
  const uint32_t bytes = ctx ? (uint32_t)__popc(loaded) * seg_bytes : (uint32_t)(L.slabs * L.rows * 128);
  const uint32_t full_cl = leader_bar<PAIR>(full);
  // completion goes to the leader's `full` (pair form of the copy) or to this
  // CTA's private `fix`
  auto issue = [&](uint32_t bar_cl, bool pair_form) {
    if (!ctx) {
      const int row = w.tile.q_start + key0;
      for (int s = 0; s < L.slabs; ++s) {
        if (pair_form)
          ptx::tma_load_3d_pair_elect(L.dst + s * L.rows * 128, L.tm_new, bar_cl, L.col0 + s * 64, w.hk, row);
        else
          ptx::tma_load_3d_elect(L.dst + s * L.rows * 128, L.tm_new, fix, L.col0 + s * 64, w.hk, row);
      }
    } else {
      if ((loaded >> lane) & 1u) {
        const int row = page * pb.p + ((key0 + lane * L.seg_rows) % pb.p);
        for (int s = 0; s < L.slabs; ++s) {
          uint8_t *d = L.dst + s * L.rows * 128 + lane * L.seg_rows * 128;
          if (pair_form)
            ptx::tma_load_3d_pair(d, L.tm_ctx, bar_cl, L.col0 + s * 64, w.hk, row);
          else
            ptx::tma_load_3d(d, L.tm_ctx, fix, L.col0 + s * 64, w.hk, row);
        }
      }
      __syncwarp();
    }
  };
  if (!need_fix) {
    if (lane == 0) {
      if constexpr (PAIR)
        ptx::mbar_arrive_expect_tx_cluster(full_cl, bytes);
      else
        ptx::mbar_arrive_expect_tx(full, bytes);
    }
    __syncwarp();
    if constexpr (PAIR) {
      issue(full_cl, true);
    } else {
      // single CTA: the plain form of the copy, completion on `full`
      if (!ctx) {
        const int row = w.tile.q_start + key0;
        for (int s = 0; s < L.slabs; ++s)
          ptx::tma_load_3d_elect(L.dst + s * L.rows * 128, L.tm_new, full, L.col0 + s * 64, w.hk, row);
      } else {
        if ((loaded >> lane) & 1u) {
          const int row = page * pb.p + ((key0 + lane * L.seg_rows) % pb.p);
          for (int s = 0; s < L.slabs; ++s)
            ptx::tma_load_3d(L.dst + s * L.rows * 128 + lane * L.seg_rows * 128, L.tm_ctx, full, L.col0 + s * 64,
                             w.hk, row);
        }
        __syncwarp();
      }
    }
    return true;
  }
  ptx::mbar_arrive_expect_tx_elect(fix, bytes);
  issue(0, false);
  // the private barrier completes even when no copy was queued
  const bool ok = wait_all3<PAIR>(sy, fix, fix_phase);
  fix_phase ^= 1u;
  if (!ok) {
    fix_pending = true;   // copies may still be in flight: drained at the end
    return false;
  }
  for (int r = lane; r < L.rows; r += 32) {
    const bool bad_row = r >= valid || (ctx && !((loaded >> (r / L.seg_rows)) & 1u));
    if (!bad_row) continue;
    for (int s = 0; s < L.slabs; ++s) {
      uint4 *z = reinterpret_cast<uint4 *>(L.dst + s * L.rows * 128 + r * 128);
#pragma unroll
      for (int q = 0; q < 8; ++q) z[q] = make_uint4(0, 0, 0, 0);
    }
  }
  ptx::fence_proxy_async_smem();
  warp_arrive_leader<PAIR>(full);
  return true;
}

// One producer warp per operand: IS_V loads V, otherwise Q and K.  Each
// fills its own stage ring as soon as the MMA warp releases a stage.
template <bool PAIR, bool IS_V, int D>
__device__ __forceinline__ void produce(const Sync &sy, const Problem &pb, const PrefillTile *tiles, int n_units,
                                        int rank, uint8_t *sQ, uint8_t *sOp, const CUtensorMap *tm_q,
                                        const CUtensorMap *tm_ctx, const CUtensorMap *tm_new) {
  using S = P3<PAIR, D>;
  constexpr int NS = IS_V ? S::NSV : S::NSK;
  Bars3 *bars = sy.bars;
  uint64_t *full = IS_V ? bars->v_full : bars->k_full;
  uint64_t *empty = IS_V ? bars->v_empty : bars->k_empty;
  uint64_t *fix = IS_V ? &bars->vfix : &bars->kfix;
  const int lane = threadIdx.x & 31;
  uint32_t fix_phase = 0;
  bool fix_pending = false;
  int gb = 0, gu = 0;
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const Unit3 w = make_unit3<PAIR>(tiles, unit_of<PAIR>(k), n_units, pb, rank);
    if (w.end) break;
    if (w.skip) continue;
    const int32_t *pt_row = pb.page_table + (size_t)w.tile.seq * pb.max_pages;
    if (!IS_V) {
      // Q of this CTA's rows, once the unit that last used the buffer has
      // finished its QKs
      const int qb = gu % S::NQ;
      if (gu >= S::NQ && !wait_all3<PAIR>(sy, &bars->q_empty[qb], (uint32_t)(((gu - S::NQ) / S::NQ) & 1))) break;
      const uint32_t qbar = leader_bar<PAIR>(&bars->q_full[qb]);
      if (lane == 0) {
        if constexpr (PAIR)
          ptx::mbar_arrive_expect_tx_cluster(qbar, S::kQBytes);
        else
          ptx::mbar_arrive_expect_tx(&bars->q_full[qb], S::kQBytes);
      }
      __syncwarp();
      // Q is read once: first out of L2, ahead of the K/V blocks that the
      // other query heads and later items of the sequence read again
      const uint64_t once = ptx::l2_evict_first_policy();
      for (int hh = 0; hh < S::D / 64; ++hh) {
        uint8_t *d = sQ + qb * S::kQBytes + hh * S::BM * 128;
        if constexpr (PAIR)
          ptx::tma_load_3d_pair_hint_elect(d, tm_q, qbar, hh * 64, w.h, w.tile.q_start + w.my_r0, once);
        else
          ptx::tma_load_3d_hint_elect(d, tm_q, &bars->q_full[qb], hh * 64, w.h, w.tile.q_start + w.my_r0, once);
      }
    }
    for (int j = 0; j < w.nb; ++j, ++gb) {
      const bool ctx = j < w.n_ctx;
      const int pos0 = ctx ? j * S::BN : (j - w.n_ctx) * S::BN;
      const int st = gb % NS;
      if (gb >= NS && !wait_all3<PAIR>(sy, &empty[st], (uint32_t)(((gb / NS) & 1) ^ 1))) {
        ok = false;
        break;
      }
      if constexpr (IS_V) {
        // keys [pos0, pos0 + BN), head-dim columns [rank * VC, + VC)
        const BlockLoad<PAIR> L{sOp + st * S::kVBytes, S::BN, S::VH, rank * S::VC, tm_ctx, tm_new, min(pb.p, S::BN)};
        ok = load_block<PAIR>(sy, pb, w, pt_row, L, ctx, pos0, &full[st], fix, fix_phase, fix_pending);
      } else {
        // keys [pos0 + rank * KH, + KH), every head-dim column
        const BlockLoad<PAIR> L{sOp + st * S::kKBytes, S::KH, S::D / 64, 0, tm_ctx, tm_new, min(pb.p, S::KH)};
        ok = load_block<PAIR>(sy, pb, w, pt_row, L, ctx, pos0 + rank * S::KH, &full[st], fix, fix_phase, fix_pending);
      }
      if (!ok) break;
    }
    ++gu;
  }
  // copies into the private barrier must land before the CTA ends (the
  // others complete on the leader's barriers, which the MMA warp or the
  // exit handshake wait for)
  if (lane == 0 && fix_pending) ptx::mbar_wait(fix, fix_phase ^ 1u);
  __syncwarp();
}

// --------------------------------------------------------- cache update
// The new K/V rows of each unit are copied into their page slots by five
// warps of the CTA: the cache-writer warp and the four epilogue warps (idle
// while a unit computes).  The G query heads of a KV head split the unit's
// rows, and the two CTAs of a pair split each share.  Warp wi of the five
// takes every fifth group of 32 16-byte chunks; each lane keeps kBatch
// chunks (and their page-table entries) in flight before storing.
constexpr int kCacheWriters = 5;

template <bool PAIR, int D>
__device__ __forceinline__ void cache_write_unit(const Problem &pb, const Unit3 &w, int rank, int wi) {
  using S = P3<PAIR, D>;
  if (!kCacheWrite) return;
  constexpr int kBatch = 4;
  constexpr int kStride = 32 * kCacheWriters;
  const int lane = threadIdx.x & 31;
  const int G = pb.hq / pb.hkv;
  constexpr int chunks = S::D / 8;
  const __nv_bfloat16 *kn = reinterpret_cast<const __nv_bfloat16 *>(pb.k_new);
  const __nv_bfloat16 *vn = reinterpret_cast<const __nv_bfloat16 *>(pb.v_new);
  __nv_bfloat16 *kc = reinterpret_cast<__nv_bfloat16 *>(pb.k_cache);
  __nv_bfloat16 *vc = reinterpret_cast<__nv_bfloat16 *>(pb.v_cache);
  const int32_t *pt_row = pb.page_table + (size_t)w.tile.seq * pb.max_pages;
  const uint64_t once = ptx::l2_evict_first_policy();
  // rows of the unit: the item (pair) or this CTA's tile
  const int u0 = PAIR ? w.tile.tile_row : w.my_r0;
  const int un = PAIR ? w.tile.rows : w.my_rows;
  const int gidx = w.h % G;
  int ra = (gidx * un) / G, rb = ((gidx + 1) * un) / G;
  if constexpr (PAIR) {
    const int len = rb - ra;
    const int a = ra + (rank * len) / 2, b = ra + ((rank + 1) * len) / 2;
    ra = a;
    rb = b;
  }
  const int total = (rb - ra) * chunks;
  for (int base = wi * 32 + lane; base < total; base += kStride * kBatch) {
    uint4 kq[kBatch], vq[kBatch];
    int pgq[kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const int idx = base + q * kStride;
      if (idx < total) {
        const int i = u0 + ra + idx / chunks;   // new-token index
        const size_t src = ((size_t)(w.tile.q_start + i) * pb.hkv + w.hk) * S::D + (idx % chunks) * 8;
        kq[q] = *reinterpret_cast<const uint4 *>(kn + src);
        vq[q] = *reinterpret_cast<const uint4 *>(vn + src);
        pgq[q] = pt_row[(w.c + i) / pb.p];
      }
    }
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const int idx = base + q * kStride;
      if (idx >= total) continue;
      const int i = u0 + ra + idx / chunks, ch = idx % chunks;
      const int pos = w.c + i;
      const int pg = pgq[q];
      if (pg < 0 || pg >= pb.num_pages) {
        if (ch == 0) atomicOr(pb.err, RPA_DEV_BAD_PAGE);
        continue;
      }
      const size_t dst = (((size_t)pg * pb.p + pos % pb.p) * pb.hkv + w.hk) * S::D + ch * 8;
      // written once and not read again by this launch: first out of L2,
      // ahead of the K/V blocks that other query heads still read
      ptx::st_global_hint(kc + dst, kq[q], once);
      ptx::st_global_hint(vc + dst, vq[q], once);
    }
  }
}

// The cache-writer warp's loop: its share (wi = 0) of every unit of the CTA.
template <bool PAIR, int D>
__device__ __forceinline__ void cache_update(const Problem &pb, const PrefillTile *tiles, int n_units, int rank) {
  for (int k = 0;; ++k) {
    const Unit3 w = make_unit3<PAIR>(tiles, unit_of<PAIR>(k), n_units, pb, rank);
    if (w.end) break;
    if (w.skip) continue;
    cache_write_unit<PAIR, D>(pb, w, rank, 0);
  }
}

// -------------------------------------------------------------- softmax
// Warpgroup `half` of the softmax turns keys [64 half, 64 half + 64) of every
// block into P; thread (row) of each warpgroup owns one query row.  The two
// threads of a row exchange their partial maxima through `red` (one mbarrier
// per warp pair and exchange parity, two elected arrivals), so both apply the
// same running max m; each keeps its own share of the row sum.  The
// reference max moves only when a block's max exceeds it by more than 2^8 (a
// lazy rescale, exact after the final 1 / l); O is then rescaled once
// PV(b - 1) is complete.
template <bool PAIR, int D>
__device__ __forceinline__ void softmax_loop(const Sync &sy, const Problem &pb, const PrefillTile *tiles,
                                             int n_units, int rank, uint32_t tmem, float *stats, float *red,
                                             float scale_log2) {
  using S = P3<PAIR, D>;
  constexpr int BN = S::BN, HK = S::HK;
  Bars3 *bars = sy.bars;
  const int warp = threadIdx.x >> 5;
  const int half = warp >> 2;
  const int wq = warp & 3;                           // warp of the pair (rows 32 wq ..)
  const int row = threadIdx.x & 127;                 // TMEM lane
  const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
  const uint32_t tO = lane_base + S::kColO + (uint32_t)(half * (S::D / 2));   // this warpgroup's half of O
  int gb = 0, gu = 0;
  int xc = 0;   // exchanges of this warp pair so far (blocks it skips have none)
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const Unit3 w = make_unit3<PAIR>(tiles, unit_of<PAIR>(k), n_units, pb, rank);
    if (w.end) break;
    if (w.skip) continue;
    const int ob = gu & 1;
    const int rn = w.my_r0 + row;                    // new-token index of this row
    const bool live = row < w.my_rows;
    float m = -INFINITY, l = 0.f, lr = 0.f;   // lr: this half's share of the normaliser of O (below)
    for (int j = 0; j < w.nb; ++j, ++gb) {
      const int sb = gb % S::NS;
      const uint32_t tS = lane_base + (uint32_t)(sb * 128);
      int lim;   // visible keys of block j for this row (a prefix of the block)
      if (!live) {
        lim = 0;
      } else if (j < w.n_ctx) {
        lim = min(BN, w.c - j * BN);
      } else {
        const int kn0 = (j - w.n_ctx) * BN;
        const int end = pb.causal ? min(w.tile.q_len, rn + 1) : w.tile.q_len;
        lim = max(0, min(BN, end - kn0));
      }
      if (!__all_sync(0xffffffffu, wait3<PAIR>(sy, &bars->s_full[sb], (uint32_t)((gb / S::NS) & 1)))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      if (__all_sync(0xffffffffu, lim == 0)) {
        // no visible key in this block for any row of the warp (the same
        // for the partner warp): P = 0, no exchange
        uint32_t z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0u;
        ptx::tmem_st32(tS + half * 32, z);
      } else {
        float x[HK];
        ptx::tmem_ld32(tS + half * HK, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
        ptx::tmem_ld32(tS + half * HK + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
        ptx::tmem_ld_wait();
        const int hl = lim - half * HK;              // visible keys of this half
        if (__any_sync(0xffffffffu, hl < HK)) {
#pragma unroll
          for (int i = 0; i < HK; ++i) x[i] = i < hl ? x[i] : -INFINITY;
        }
        float mq[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
        for (int i = 4; i < HK; i += 8) {
          mq[0] = ptx::fmax3(mq[0], x[i], x[i + 1]);
          mq[1] = ptx::fmax3(mq[1], x[i + 2], x[i + 3]);
          if (i + 4 < HK) {
            mq[2] = ptx::fmax3(mq[2], x[i + 4], x[i + 5]);
            mq[3] = ptx::fmax3(mq[3], x[i + 6], x[i + 7]);
          }
        }
        const float mine = ptx::fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3]));
        float *rb = red + (xc & 1) * 2 * S::BM;
        rb[half * S::BM + row] = mine;
        __syncwarp();
        if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(&bars->xch[wq][xc & 1]);
        if (!__all_sync(0xffffffffu, wait3<PAIR>(sy, &bars->xch[wq][xc & 1], (uint32_t)((xc >> 1) & 1)))) {
          ok = false;
          break;
        }
        ++xc;
        const float mx = fmaxf(mine, rb[(half ^ 1) * S::BM + row]) * scale_log2;
        const float m_new = fmaxf(m, mx);
        const bool need = m != -INFINITY && m_new > m + kRescaleThreshold;
        float alpha = 1.f;
        if (__any_sync(0xffffffffu, need)) {
          // O holds the unit's blocks up to j - 1: wait for PV(gb - 1) (and
          // so PV(gb - 2); PV(gb - 3) is complete, since S(gb) is); each
          // warpgroup rescales its half of O's columns
          alpha = (m_new == m) ? 1.f : ptx::ex2(m - m_new);
          if (j > 0) {
            if (!__all_sync(0xffffffffu,
                            wait3<PAIR>(sy, &bars->pv_done[(gb - 1) & 1], (uint32_t)(((gb - 1) >> 1) & 1)))) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < S::D / 64; ++cc) {
              uint32_t r[32];
              ptx::tmem_ld32(tO + cc * 32, r);
              ptx::tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
              ptx::tmem_st32(tO + cc * 32, r);
            }
          }
          m = m_new;
        } else if (m == -INFINITY) {
          m = m_new;
        }
        const float neg_m = m == -INFINITY ? 0.f : -m;
        const uint64_t scale2 = ptx::f2_pack(scale_log2, scale_log2);
        const uint64_t negm2 = ptx::f2_pack(neg_m, neg_m);
        uint64_t sp2[4] = {0, 0, 0, 0};
        uint32_t pk[32];   // P of this half's 64 keys as bf16 pairs: columns [32 half, 32 half + 32)
#pragma unroll
        for (int i = 0; i < HK; i += 2) {
          float a0, a1;
          ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(x[i], x[i + 1]), scale2, negm2), a0, a1);
          const uint64_t pp = ptx::f2_pack(ptx::ex2(a0), ptx::ex2(a1));
          sp2[(i >> 1) & 3] = ptx::f2_add(sp2[(i >> 1) & 3], pp);
          float p0, p1;
          ptx::f2_unpack(pp, p0, p1);
          pk[i >> 1] = ptx::pack_bf16(p0, p1);
        }
        ptx::tmem_st32(tS + half * 32, pk);
        float sp[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) ptx::f2_unpack(sp2[q], sp[2 * q], sp[2 * q + 1]);
        const float sum = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
        // The PV MMA takes P rounded to bf16.  Under the lazy rescale the
        // largest weight of this half-block can be up to 2^8 (not exactly
        // 1), and its rounding (relative 2^-9) moves O by up to 2^-9 |V|
        // when one key dominates the row.  lr, the normaliser of O,
        // therefore counts that weight as rounded, so that its rounding
        // cancels in O / lr; the other weights keep the error of a kernel
        // whose max weight is 1.  l keeps the exact fp32 sum, for lse.
        const float pmax = ptx::ex2(fmaf(mine, scale_log2, neg_m));   // as the loop computed it
        l = l * alpha + sum;
        lr = lr * alpha + (sum - (pmax - ptx::round_bf16(pmax)));
      }
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      warp_arrive_leader<PAIR>(&bars->p_full[sb]);
    }
    if (!ok) break;
    // row statistics of the unit for the epilogue
    if (gu >= 2 && !__all_sync(0xffffffffu, wait3<PAIR>(sy, &bars->st_free[ob], (uint32_t)(((gu - 2) >> 1) & 1)))) {
      ok = false;
      break;
    }
    stats[(ob * 5 + half) * S::BM + row] = l;
    stats[(ob * 5 + 3 + half) * S::BM + row] = lr;
    if (half == 0) stats[(ob * 5 + 2) * S::BM + row] = m;
    ptx::mbar_arrive(&bars->st_full[ob]);
    ++gu;
  }
}

// ------------------------------------------------------------- epilogue
template <bool PAIR, int D>
__device__ __forceinline__ void epilogue_loop(const Sync &sy, const Problem &pb, const PrefillTile *tiles,
                                              int n_units, int rank, uint32_t tmem, const float *stats) {
  using S = P3<PAIR, D>;
  Bars3 *bars = sy.bars;
  const int warp = threadIdx.x >> 5;
  const int row = threadIdx.x & 127;
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  int gu = 0;
  for (int k = 0;; ++k) {
    const Unit3 w = make_unit3<PAIR>(tiles, unit_of<PAIR>(k), n_units, pb, rank);
    if (w.end) break;
    if (w.skip) continue;
    // this warp's share of the unit's cache update, while the unit computes
    cache_write_unit<PAIR, D>(pb, w, rank, 1 + (warp & 3));
    const int ob = gu & 1;
    const uint32_t ph = (uint32_t)((gu >> 1) & 1);
    if (!__all_sync(0xffffffffu, wait3<PAIR>(sy, &bars->o_full, (uint32_t)(gu & 1)))) break;
    if (!__all_sync(0xffffffffu, wait3<PAIR>(sy, &bars->st_full[ob], ph))) break;
    ptx::tc_fence_after();
    const float l = stats[(ob * 5 + 0) * S::BM + row] + stats[(ob * 5 + 1) * S::BM + row];
    const float lr = stats[(ob * 5 + 3) * S::BM + row] + stats[(ob * 5 + 4) * S::BM + row];
    const float m = stats[(ob * 5 + 2) * S::BM + row];
    ptx::mbar_arrive(&bars->st_free[ob]);
    // O a 32-column chunk at a time into registers, scaled by 1 / l and
    // stored; released after the last chunk (its next writer, the next
    // unit's first PV, is queued two blocks behind that unit's QKs)
    const bool store = row < w.my_rows;
    const int rn = w.my_r0 + row;
    const float inv = store ? 1.f / lr : 0.f;
    const uint64_t once = ptx::l2_evict_first_policy();   // outputs are written once: first out of L2
    uint4 *out = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(pb.out) +
                                           ((size_t)(w.tile.q_start + (store ? rn : 0)) * pb.hq + w.h) * S::D);
#pragma unroll 1
    for (int cc = 0; cc < S::D / 32; ++cc) {
      uint32_t ov[32];
      ptx::tmem_ld32(lane_base + S::kColO + cc * 32, ov);
      ptx::tmem_ld_wait();
      if (store) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t o2[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            o2[i] = ptx::pack_bf16(__uint_as_float(ov[q * 8 + 2 * i]) * inv, __uint_as_float(ov[q * 8 + 2 * i + 1]) * inv);
          ptx::st_global_hint(out + cc * 4 + q, make_uint4(o2[0], o2[1], o2[2], o2[3]), once);
        }
      }
    }
    ptx::tc_fence_before();
    warp_arrive_leader<PAIR>(&bars->o_free);
    if (store && pb.lse != nullptr) pb.lse[(size_t)(w.tile.q_start + rn) * pb.hq + w.h] = (m + log2f(l)) * kLn2;
    ++gu;
  }
}

// --------------------------------------------------------------- kernel
template <bool PAIR, int D>
__global__ void __launch_bounds__(512, 1)
    prefill3_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                    const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kn,
                    const __grid_constant__ CUtensorMap tm_vn, const Problem pb,
                    const PrefillTile *__restrict__ tiles, int n_units, float scale_log2) {
  using S = P3<PAIR, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = base;                     // Q buffer b at sQ + b * kQBytes
  uint8_t *sK = sQ + S::NQ * S::kQBytes;
  uint8_t *sV = sK + S::NSK * S::kKBytes;
  float *stats = reinterpret_cast<float *>(base + S::kData);
  float *red = stats + S::kStatFloats;
  Bars3 *bars = reinterpret_cast<Bars3 *>(red + S::kRedFloats);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int rank = PAIR ? (int)ptx::cluster_ctarank() : 0;
  if (pb.dev_counts != nullptr) {
    // capacity-sized grid: groups without a unit leave before any set-up
    // (both CTAs of a pair decide alike)
    const int units = pb.dev_counts[kCntPrefill] * (PAIR ? pb.hq : 2 * pb.hq);
    if (group_id<PAIR>() >= units) return;
    if (units < n_units) n_units = units;
  }

  if (tid == 0) {
    constexpr uint32_t nc = S::NCTA;
    for (int i = 0; i < 3; ++i) {
      ptx::mbar_init(&bars->s_full[i], 1);
      ptx::mbar_init(&bars->p_full[i], S::kSoftmaxArrivals);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->q_full[i], nc);
      ptx::mbar_init(&bars->q_empty[i], 1);
      ptx::mbar_init(&bars->pv_done[i], 1);
      ptx::mbar_init(&bars->st_full[i], 256);
      ptx::mbar_init(&bars->st_free[i], 128);
      for (int q = 0; q < 4; ++q) ptx::mbar_init(&bars->xch[q][i], 2);
    }
    ptx::mbar_init(&bars->o_full, 1);
    ptx::mbar_init(&bars->o_free, S::kEpilogueArrivals);
    for (int i = 0; i < S::NSK; ++i) {
      ptx::mbar_init(&bars->k_full[i], nc);
      ptx::mbar_init(&bars->k_empty[i], 1);
    }
    for (int i = 0; i < S::NSV; ++i) {
      ptx::mbar_init(&bars->v_full[i], nc);
      ptx::mbar_init(&bars->v_empty[i], 1);
    }
    ptx::mbar_init(&bars->kfix, 1);
    ptx::mbar_init(&bars->vfix, 1);
    ptx::mbar_init(&bars->drain, 1);
    ptx::mbar_init(&bars->exit_bar, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 13) {
    if constexpr (PAIR) {
      ptx::tmem_alloc_pair(tmem_slot, S::kTmemCols);
      ptx::tmem_relinquish_pair();
    } else {
      ptx::tmem_alloc(tmem_slot, S::kTmemCols);
      ptx::tmem_relinquish();
    }
  }
  if (warp == 12 && (tid & 31) == 0) {
    ptx::tma_prefetch_desc(&tm_q);
    ptx::tma_prefetch_desc(&tm_kc);
    ptx::tma_prefetch_desc(&tm_vc);
    ptx::tma_prefetch_desc(&tm_kn);
    ptx::tma_prefetch_desc(&tm_vn);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {
    // both CTAs' barriers are initialised before either side signals the other
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  }
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Sync sy{bars, abort_flag, PAIR ? ptx::mapa_shared((const void *)abort_flag, (uint32_t)(rank ^ 1)) : 0u, pb.err};

  if (warp >= 12) {
    if (warp == 12) {
      produce<PAIR, false, D>(sy, pb, tiles, n_units, rank, sQ, sK, &tm_q, &tm_kc, &tm_kn);
    } else if (warp == 14) {
      produce<PAIR, true, D>(sy, pb, tiles, n_units, rank, sQ, sV, &tm_q, &tm_vc, &tm_vn);
    } else if (warp == 13) {
      if (rank == 0) {
        mma_loop<PAIR, D>(sy, pb, tiles, n_units, tmem, ptx::smem_u32(sQ), ptx::smem_u32(sK), ptx::smem_u32(sV));
        // every MMA this warp issued is complete before the CTA (and, through
        // the exit handshake below, its peer) releases TMEM or leaves
        commit<PAIR>(&bars->drain);
        if ((tid & 31) == 0) ptx::mbar_wait(&bars->drain, 0);
        __syncwarp();
      }
    } else {
      cache_update<PAIR, D>(pb, tiles, n_units, rank);
    }
  } else if (warp < 8) {
    softmax_loop<PAIR, D>(sy, pb, tiles, n_units, rank, tmem, stats, red, scale_log2);
  } else {
    epilogue_loop<PAIR, D>(sy, pb, tiles, n_units, rank, tmem, stats);
  }

  ptx::tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {
    // neither CTA frees its TMEM or shared memory while the other may still
    // signal it: each tells the other it is done and waits to be told
    if (tid == 0) {
      ptx::mbar_arrive_cluster(ptx::mapa_shared(&bars->exit_bar, (uint32_t)(rank ^ 1)));
      ptx::mbar_wait(&bars->exit_bar, 0);
    }
    __syncthreads();
  }
  ptx::tc_fence_after();
  if (warp == 13) {
    if constexpr (PAIR)
      ptx::tmem_dealloc_pair(tmem, S::kTmemCols);
    else
      ptx::tmem_dealloc(tmem, S::kTmemCols);
  }
}

template <bool PAIR, int D>
cudaError_t launch_t(const Problem &pb, const PrefillTile *tiles, int n_tiles, int max_ctas, cudaStream_t stream) {
  using S = P3<PAIR, D>;
  CUtensorMap tq, tkc, tvc, tkn, tvn;
  const uint64_t qdims[3] = {(uint64_t)S::D, (uint64_t)pb.hq, (uint64_t)pb.total_q};
  const uint64_t qstr[2] = {(uint64_t)S::D * 2, (uint64_t)pb.hq * S::D * 2};
  const uint32_t qbox[3] = {64, 1, (uint32_t)S::BM};
  const uint64_t cdims[3] = {(uint64_t)S::D, (uint64_t)pb.hkv, (uint64_t)pb.num_pages * pb.p};
  const uint64_t cstr[2] = {(uint64_t)S::D * 2, (uint64_t)pb.hkv * S::D * 2};
  const uint32_t kcbox[3] = {64, 1, (uint32_t)(pb.p < S::KH ? pb.p : S::KH)};
  const uint32_t vcbox[3] = {64, 1, (uint32_t)(pb.p < S::BN ? pb.p : S::BN)};
  const uint64_t ndims[3] = {(uint64_t)S::D, (uint64_t)pb.hkv, (uint64_t)pb.total_q};
  const uint64_t nstr[2] = {(uint64_t)S::D * 2, (uint64_t)pb.hkv * S::D * 2};
  const uint32_t knbox[3] = {64, 1, (uint32_t)S::KH};
  const uint32_t vnbox[3] = {64, 1, (uint32_t)S::BN};
  if (!make_tmap_bf16_3d(&tq, pb.q, qdims, qstr, qbox, true) ||
      !make_tmap_bf16_3d(&tkc, pb.k_cache, cdims, cstr, kcbox, true) ||
      !make_tmap_bf16_3d(&tvc, pb.v_cache, cdims, cstr, vcbox, true) ||
      !make_tmap_bf16_3d(&tkn, pb.k_new, ndims, nstr, knbox, true) ||
      !make_tmap_bf16_3d(&tvn, pb.v_new, ndims, nstr, vnbox, true))
    return cudaErrorInvalidValue;
  auto kern = prefill3_kernel<PAIR, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem);
  if (e != cudaSuccess) return e;
  const int n_units = n_tiles * (PAIR ? pb.hq : 2 * pb.hq);
  // resident groups: SMs (single CTAs), or co-resident clusters of two
  static int groups_cap[2] = {0, 0};
  int &cap = groups_cap[PAIR ? 1 : 0];
  if (cap == 0) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0)
      sms = 148;
    cap = sms;
    if constexpr (PAIR) {
      cudaLaunchConfig_t qc = {};
      cudaLaunchAttribute qa[1];
      qa[0].id = cudaLaunchAttributeClusterDimension;
      qa[0].val.clusterDim.x = 2;
      qa[0].val.clusterDim.y = 1;
      qa[0].val.clusterDim.z = 1;
      qc.gridDim = dim3((unsigned)(2 * (sms / 2)), 1, 1);
      qc.blockDim = dim3(512, 1, 1);
      qc.dynamicSmemBytes = S::kSmem;
      qc.attrs = qa;
      qc.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kern, &qc) != cudaSuccess || clusters <= 0) {
        cudaGetLastError();
        clusters = sms / 2;
      }
      cap = clusters;
    }
  }
  int groups = n_units < cap ? n_units : cap;
  const int max_groups = max_ctas > 0 ? (PAIR ? max_ctas / 2 : max_ctas) : 0;
  if (max_groups > 0 && groups > max_groups) groups = max_groups;
  if (groups < 1) groups = 1;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3((unsigned)(groups * S::NCTA), 1, 1);
  cfg.blockDim = dim3(512, 1, 1);
  cfg.dynamicSmemBytes = S::kSmem;
  cfg.stream = stream;
  if constexpr (PAIR) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  e = cudaLaunchKernelEx(&cfg, kern, tq, tkc, tvc, tkn, tvn, pb, tiles, n_units, pb.scale * kLog2e);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill3(const Problem &pb, const PrefillTile *tiles, int n_tiles, int max_ctas, bool pair,
                            cudaStream_t stream) {
  if (n_tiles <= 0) return cudaSuccess;
  if (pb.d == 128)
    return pair ? launch_t<true, 128>(pb, tiles, n_tiles, max_ctas, stream)
                : launch_t<false, 128>(pb, tiles, n_tiles, max_ctas, stream);
  if (pb.d == 256 && pair) return launch_t<true, 256>(pb, tiles, n_tiles, max_ctas, stream);
  return cudaErrorInvalidValue;
}

}  // namespace rpa
