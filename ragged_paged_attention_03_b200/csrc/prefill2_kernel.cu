// prefill2_kernel.cu -- prefill / chunked-prefill attention for head_dim <= 128
// with two 128-row query tiles per CTA sharing every K/V block, so that one
// tile's softmax runs while the tensor cores work on the other tile (the
// compute-bound regime of the RPA talk summary, 00:11:09), and the fused
// cache update of 00:06:36.
//
// Roles (384 threads launched at 168 registers = 64512; setmaxnreg moves the
// softmax warpgroups to 200 and the rest to 96: 256*200 + 128*96 = 63488):
//   warpgroup 0 (warps 0-3)  softmax + epilogue of tile 0 (one row per thread)
//   warpgroup 1 (warps 4-7)  softmax + epilogue of tile 1
//   warp 8                   TMA producer: Q tiles, then K/V blocks of 128
//                            keys (context from pages, new tokens from
//                            k_new / v_new; rows without a valid key zeroed)
//   warp 9                   TMEM owner and MMA issue
//   warps 10-11              fused cache update: this CTA's share of the new
//                            K/V rows copied into their page slots
// A second role layout (the `split` argument) gives V a producer of its own in
// warp 10, leaving warp 11 to the cache update: the planner picks it for batches
// whose prefill work is mostly paged context (latency-bound gathers, few new
// rows to write), the first one otherwise.
// The producer and MMA warps run their loops with all 32 lanes and let one
// elected lane issue each TMA copy, MMA, commit and arrive: a single-lane
// branch would keep the operands in per-thread registers and cost many issue
// slots per MMA while the softmax warps keep the sub-partitions busy.
//
// TMEM (512 columns): S/P of tile 0 | S/P of tile 1 | O of tile 0 | O of tile 1.
// P overwrites its tile's S as bf16 and is the A operand of O += P V.  The
// tensor pipe sees QK(0,j+1), PV(1,j), QK(1,j+1), PV(0,j+1), ...: while one
// tile's softmax runs, the other tile's PV and QK execute.
//
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
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct P2Shape {
  static constexpr int BM = 128;     // rows per tile, two tiles per CTA
  static constexpr int BN = 128;     // keys per block
  // K and V have rings of their own: a K stage is released two MMA groups
  // before the V stage of the same block, and the next block needs K first.
  static constexpr int NSK = D == 64 ? 4 : 3;
  static constexpr int NSV = D == 64 ? 4 : 2;
  static constexpr int kHalves = D / 64;
  static constexpr int kQBytes = kHalves * BM * 128;
  static constexpr int kKVBytes = kHalves * BN * 128;
  static constexpr int kData = 2 * kQBytes + (NSK + NSV) * kKVBytes;
  static constexpr int kSmem = 1024 + kData + 512;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 256;   // O of tile t at kColO + t * D
};

struct Bars2 {
  uint64_t q_full, q_empty;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], p_full[2], pv_done[2], o_free[2];
  uint64_t p_half[2];   // P of keys 0..63 stored (PV's first four k-steps may start)
  uint64_t fix[2], drain;   // fix[1]: the V producer's, when V has its own warp
};

__device__ __forceinline__ bool wait_bar2(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
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

// wait_bar2 by every lane of a warp, with a warp-uniform result.
__device__ __forceinline__ bool wait_all(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint32_t *err) {
  return __all_sync(0xffffffffu, wait_bar2(bar, parity, abort_flag, err));
}

__device__ __forceinline__ void setmaxnreg_inc200() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 200;" ::: "memory");
}
__device__ __forceinline__ void setmaxnreg_dec96() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 96;" ::: "memory");
}

// Unit order of a persistent CTA: round r takes unit r * G + b on even
// rounds and r * G + (G - 1 - b) on odd ones ("snake"), so that with the
// units sorted heaviest first every CTA gets a similar share of the work.
__device__ __forceinline__ int unit_of(int r) {
  const int G = gridDim.x, b = blockIdx.x;
  return r * G + ((r & 1) ? G - 1 - b : b);
}

// Geometry of one work unit (a 256-row item of one sequence, one query head).
struct Unit {
  PrefillTile tile;
  int h, hk, c, r0, n_ctx, nb;
  int rows_t[2], n_t[2];
};

// Tile descriptor of unit u, or an empty one (rows == 0) past the last
// unit.  Each role loads the next unit's descriptor at the top of the
// current unit, so that a unit change does not start with a dependent
// global read of the plan.
__device__ __forceinline__ PrefillTile load_tile(const PrefillTile *tiles, int u, int n_units, int hq) {
  PrefillTile t{};
  if (u < n_units) t = tiles[u / hq];
  return t;
}

template <int BM, int BN>
__device__ __forceinline__ Unit make_unit(const PrefillTile &tile, int u, const Problem &pb) {
  Unit w;
  w.tile = tile;
  w.h = u % pb.hq;
  w.hk = w.h / (pb.hq / pb.hkv);
  w.c = w.tile.kv_len - w.tile.q_len;
  w.r0 = w.tile.tile_row;
  w.rows_t[0] = min(BM, w.tile.rows);
  w.rows_t[1] = max(0, w.tile.rows - BM);
  w.n_ctx = (w.c + BN - 1) / BN;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int new_end = pb.causal ? w.r0 + t * BM + w.rows_t[t] : w.tile.q_len;
    w.n_t[t] = w.rows_t[t] == 0 ? 0 : w.n_ctx + (new_end + BN - 1) / BN;
  }
  w.nb = max(w.n_t[0], w.n_t[1]);
  return w;
}

// QK(t, gblk): S of tile t = Q_t K^T for K/V block gblk (K stage gblk % NSK).
template <int D>
__device__ __forceinline__ bool issue_qk(Bars2 *bars, volatile int *abort_flag, uint32_t *err, uint32_t tS,
                                         uint64_t dq, uint64_t dk0, int gblk, bool wait_k) {
  using S = P2Shape<D>;
  constexpr uint32_t idesc = ptx::umma_idesc_bf16(128, S::BN, false);
  const int s = gblk % S::NSK;
  if (wait_k && !wait_all(&bars->k_full[s], (uint32_t)((gblk / S::NSK) & 1), abort_flag, err)) return false;
  ptx::tc_fence_after();
  const uint64_t dk = dk0 + (uint64_t)((s * S::kKVBytes) >> 4);
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const uint32_t offq = ((ks >> 2) * S::BM * 128 + (ks & 3) * 32) >> 4;
    const uint32_t offk = ((ks >> 2) * S::BN * 128 + (ks & 3) * 32) >> 4;
    ptx::umma_ss_elect(tS, dq + offq, dk + offk, idesc, ks > 0 ? 1u : 0u);
  }
  return true;
}

// PV(t, gblk): O_t (+)= P_t V for K/V block gblk; P_t is read from TMEM.
template <int D>
__device__ __forceinline__ bool issue_pv(Bars2 *bars, volatile int *abort_flag, uint32_t *err, int t,
                                         uint32_t tS, uint32_t tO, uint64_t dv0, int gblk, int tblk,
                                         bool first, bool wait_v) {
  using S = P2Shape<D>;
  constexpr uint32_t idesc = ptx::umma_idesc_bf16(128, D, true);
  const int s = gblk % S::NSV;
  // P arrives in two halves: keys 0..63 feed the first four k-steps while
  // the softmax warps still compute the rest
  if (!wait_all(&bars->p_half[t], (uint32_t)(tblk & 1), abort_flag, err)) return false;
  if (wait_v && !wait_all(&bars->v_full[s], (uint32_t)((gblk / S::NSV) & 1), abort_flag, err)) return false;
  ptx::tc_fence_after();
  const uint64_t dv = dv0 + (uint64_t)((s * S::kKVBytes) >> 4);
#pragma unroll
  for (int kk = 0; kk < S::BN / 32; ++kk)
    ptx::umma_ts_elect(tO, tS + kk * 8, dv + (uint64_t)((kk * 16 * 128) >> 4), idesc, (!first || kk > 0) ? 1u : 0u);
  if (!wait_all(&bars->p_full[t], (uint32_t)(tblk & 1), abort_flag, err)) return false;
  ptx::tc_fence_after();
#pragma unroll
  for (int kk = S::BN / 32; kk < S::BN / 16; ++kk)
    ptx::umma_ts_elect(tO, tS + kk * 8, dv + (uint64_t)((kk * 16 * 128) >> 4), idesc, 1u);
  return true;
}

// The MMA warp (all 32 lanes; one elected lane issues).  Per unit, with the
// two tiles' chains interleaved (the tensor pipe sees QK0, PV1, QK1, PV0,
// ...):
//   prologue  QK(0,0) QK(1,0) PV(0,0)
//   block j   QK(0,j+1) PV(1,j) QK(1,j+1) PV(0,j+1)
// A QK into tile t's S/P columns is issued right after the PV that reads P
// from them, without waiting for that PV to finish: tcgen05.mma operations
// issued by one thread execute in issue order.  The same order makes
// s_full(t, j+1) (committed after QK(t, j+1)) imply that PV(t, j) is
// complete, which the softmax warps rely on before rescaling O.
template <int D>
__device__ __forceinline__ void mma_loop(Bars2 *bars, volatile int *abort_flag, const Problem pb,
                                         const PrefillTile *tiles, int n_units, uint32_t tmem, uint32_t q_addr,
                                         uint32_t k_addr, uint32_t v_addr) {
  using S = P2Shape<D>;
  constexpr int BM = S::BM, BN = S::BN, NSK = S::NSK, NSV = S::NSV;
  const uint32_t tS0 = tmem, tS1 = tmem + 128;
  const uint32_t tO0 = tmem + S::kColO, tO1 = tmem + S::kColO + D;
  // Descriptors of the stage-0 / tile-0 operands; the start-address field
  // is the low 14 bits (address / 16), so stages, tiles, k-steps and column
  // tiles are reached by adding (byte offset / 16).
  const uint64_t dq0 = ptx::umma_desc_sw128(q_addr, 16, 1024);
  const uint64_t dq1 = dq0 + (uint64_t)(S::kQBytes >> 4);
  const uint64_t dk0 = ptx::umma_desc_sw128(k_addr, 16, 1024);
  const uint64_t dv0 = ptx::umma_desc_sw128(v_addr, BN * 128, 1024);
  uint32_t *err = pb.err;
  int g0 = 0, gt0 = 0, gt1 = 0, ep0 = 0, ep1 = 0, uq = 0;
  bool ok = true;
  PrefillTile next = load_tile(tiles, unit_of(0), n_units, pb.hq);
  for (int r = 0, u = unit_of(0); ok && u < n_units; u = unit_of(++r), ++uq) {
    const Unit w = make_unit<BM, BN>(next, u, pb);
    next = load_tile(tiles, unit_of(r + 1), n_units, pb.hq);
    if (w.tile.rows == 0) break;   // end of a device-planned tile list
    const int n0 = w.n_t[0], n1 = w.n_t[1], nb = w.nb;
    ok = wait_all(&bars->q_full, (uint32_t)(uq & 1), abort_flag, err);
    // prologue
    if (ok && n0 > 0) ok = issue_qk<D>(bars, abort_flag, err, tS0, dq0, dk0, g0, true);
    if (ok && n0 > 0) ptx::umma_commit_elect(&bars->s_full[0]);
    if (ok && n1 > 0) ok = issue_qk<D>(bars, abort_flag, err, tS1, dq1, dk0, g0, n0 == 0);
    if (ok && n1 > 0) ptx::umma_commit_elect(&bars->s_full[1]);
    if (ok) ptx::umma_commit_elect(&bars->k_empty[g0 % NSK]);
    if (ok && nb == 1) ptx::umma_commit_elect(&bars->q_empty);
    if (ok && n0 > 0) {
      // O_0 is overwritten by the unit's first PV: the softmax warps must
      // have read the previous unit's O_0
      if (ep0 > 0) ok = wait_all(&bars->o_free[0], (uint32_t)((ep0 - 1) & 1), abort_flag, err);
      if (ok) ok = issue_pv<D>(bars, abort_flag, err, 0, tS0, tO0, dv0, g0, gt0, true, true);
      // pv_done is waited for only after a tile's last block (epilogue)
      if (ok && n0 == 1) ptx::umma_commit_elect(&bars->pv_done[0]);
    }
    for (int j = 0; ok && j < nb; ++j) {
      const bool k_next_waited = j + 1 < n0;
      if (j + 1 < n0) {
        ok = issue_qk<D>(bars, abort_flag, err, tS0, dq0, dk0, g0 + j + 1, true);
        if (ok) ptx::umma_commit_elect(&bars->s_full[0]);
      }
      if (ok && j < n1) {
        if (j == 0 && ep1 > 0) ok = wait_all(&bars->o_free[1], (uint32_t)((ep1 - 1) & 1), abort_flag, err);
        // V(j) was already waited for by PV(0, j) when tile 0 used block j
        if (ok) ok = issue_pv<D>(bars, abort_flag, err, 1, tS1, tO1, dv0, g0 + j, gt1 + j, j == 0, j >= n0);
        if (ok && j + 1 == n1) ptx::umma_commit_elect(&bars->pv_done[1]);
      }
      if (ok) ptx::umma_commit_elect(&bars->v_empty[(g0 + j) % NSV]);   // both PVs of block j issued
      if (ok && j + 1 < n1) {
        ok = issue_qk<D>(bars, abort_flag, err, tS1, dq1, dk0, g0 + j + 1, !k_next_waited);
        if (ok) ptx::umma_commit_elect(&bars->s_full[1]);
      }
      if (ok && j + 1 < nb) ptx::umma_commit_elect(&bars->k_empty[(g0 + j + 1) % NSK]);
      if (ok && j + 2 == nb) ptx::umma_commit_elect(&bars->q_empty);   // last QK of the unit issued
      if (ok && j + 1 < n0) {
        ok = issue_pv<D>(bars, abort_flag, err, 0, tS0, tO0, dv0, g0 + j + 1, gt0 + j + 1, false, true);
        if (ok && j + 2 == n0) ptx::umma_commit_elect(&bars->pv_done[0]);
      }
    }
    g0 += nb;
    gt0 += n0;
    gt1 += n1;
    ep0 += n0 > 0 ? 1 : 0;
    ep1 += n1 > 0 ? 1 : 0;
  }
  ptx::umma_commit_elect(&bars->drain);
  ptx::mbar_wait(&bars->drain, 0);
  __syncwarp();
}

// One producer warp for both operands: for every block, K as soon as its
// stage is free, then V.  The Q tiles of each unit first.  Context blocks are
// gathered one page segment per box through the page table (block j+1's
// entries are read while block j is issued); a block with rows that hold no
// valid key (past the context or the sequence, or on a page outside the
// pool) goes through a private barrier: the copies land, the rows are zeroed,
// then the block is published.
template <int D>
__device__ __forceinline__ void produce_kv(Bars2 *bars, volatile int *abort_flag, const Problem pb,
                                           const PrefillTile *tiles, int n_units, uint8_t *sQ, uint8_t *sK,
                                           uint8_t *sV, const CUtensorMap *tmq, const CUtensorMap *tmkc,
                                           const CUtensorMap *tmvc, const CUtensorMap *tmkn, const CUtensorMap *tmvn) {
  using S = P2Shape<D>;
  constexpr int BM = S::BM, BN = S::BN, NSK = S::NSK, NSV = S::NSV;
  const CUtensorMap &tm_q = *tmq, &tm_kc = *tmkc, &tm_vc = *tmvc, &tm_kn = *tmkn, &tm_vn = *tmvn;
  const int lane = threadIdx.x & 31;
  // Q tiles are read once: first out of L2, ahead of the K/V blocks that
  // the other query heads of the KV head read again
  const uint64_t once = ptx::l2_evict_first_policy();
  const int br = pb.p < BN ? pb.p : BN;
  const int nseg = BN / br;
  uint32_t fix_phase = 0;
  int g = 0;            // K/V blocks started so far (all units)
  int gk = 0, gv = 0;   // blocks whose K (V) copies were queued and published
  bool fix_pending = false;
  int uq = 0;           // units started
  bool ok = true;
  PrefillTile next = load_tile(tiles, unit_of(0), n_units, pb.hq);
  for (int r = 0, u = unit_of(0); ok && u < n_units; u = unit_of(++r), ++uq) {
    const Unit w = make_unit<BM, BN>(next, u, pb);
    next = load_tile(tiles, unit_of(r + 1), n_units, pb.hq);
    if (w.tile.rows == 0) break;   // end of a device-planned tile list
    const int32_t *pt_row = pb.page_table + (size_t)w.tile.seq * pb.max_pages;
    // Q of both tiles, once the previous unit's QK MMAs are done with sQ
    if (uq > 0 && !wait_all(&bars->q_empty, (uint32_t)((uq - 1) & 1), abort_flag, pb.err)) break;
    ptx::mbar_arrive_expect_tx_elect(&bars->q_full, (w.rows_t[1] > 0 ? 2 : 1) * S::kQBytes);
    for (int t = 0; t < 2; ++t) {
      if (w.rows_t[t] == 0) continue;
      for (int hh = 0; hh < S::kHalves; ++hh)
        ptx::tma_load_3d_hint_elect(sQ + t * S::kQBytes + hh * BM * 128, &tm_q, &bars->q_full, hh * 64, w.h,
                                    w.tile.q_start + w.r0 + t * BM, once);
    }
    // page of this lane's segment of context block j (-1: no segment);
    // block j+1's entries are read while block j is issued
    auto page_of = [&](int j) -> int {
      const int sp = j * BN + lane * br;
      return (j < w.n_ctx && lane < nseg && sp < w.c) ? pt_row[sp / pb.p] : -1;
    };
    int page_next = page_of(0);
    for (int j = 0; j < w.nb; ++j, ++g) {
      const int page = page_next;
      if (j + 1 < w.nb) page_next = page_of(j + 1);
      const int sk = g % NSK, sv = g % NSV;
      const uint32_t phk = (uint32_t)((g / NSK) & 1), phv = (uint32_t)((g / NSV) & 1);
      uint8_t *dk = sK + sk * S::kKVBytes;
      uint8_t *dv = sV + sv * S::kKVBytes;
      const bool ctx = j < w.n_ctx;
      const int pos0 = ctx ? j * BN : (j - w.n_ctx) * BN;
      const int valid = min(BN, (ctx ? w.c : w.tile.q_len) - pos0);
      bool seg_loaded = false, seg_bad = false;
      if (ctx && lane < nseg && pos0 + lane * br < w.c) {
        if (page < 0 || page >= pb.num_pages) {
          seg_bad = true;
          atomicOr(pb.err, RPA_DEV_BAD_PAGE);
        } else {
          seg_loaded = true;
        }
      }
      const unsigned loaded_mask = __ballot_sync(0xffffffffu, seg_loaded);
      const bool fix = valid < BN || __any_sync(0xffffffffu, seg_bad);
      const uint32_t seg_bytes = (uint32_t)(S::kHalves * br * 128);
      const uint32_t blk_bytes = ctx ? (uint32_t)__popc(loaded_mask) * seg_bytes : (uint32_t)S::kKVBytes;
      // the copies of one operand (K or V) of this block into dst
      auto load = [&](uint8_t *dst, const CUtensorMap *tm_new, const CUtensorMap *tm_ctx, uint64_t *bar) {
        if (!ctx) {
          const int row = w.tile.q_start + pos0;
          for (int hh = 0; hh < S::kHalves; ++hh)
            ptx::tma_load_3d_elect(dst + hh * BN * 128, tm_new, bar, hh * 64, w.hk, row);
        } else {
          // each lane queues the copies of its own page segment, so one
          // instruction covers every segment of the block
          if ((loaded_mask >> lane) & 1u) {
            const int row = page * pb.p + ((pos0 + lane * br) % pb.p);
            for (int hh = 0; hh < S::kHalves; ++hh)
              ptx::tma_load_3d(dst + hh * BN * 128 + lane * br * 128, tm_ctx, bar, hh * 64, w.hk, row);
          }
          __syncwarp();
        }
      };
      if (!fix) {
        // K as soon as its stage is free, then V
        if (g >= NSK && !wait_all(&bars->k_empty[sk], phk ^ 1u, abort_flag, pb.err)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx_elect(&bars->k_full[sk], blk_bytes);
        load(dk, &tm_kn, &tm_kc, &bars->k_full[sk]);
        ++gk;
        if (g >= NSV && !wait_all(&bars->v_empty[sv], phv ^ 1u, abort_flag, pb.err)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx_elect(&bars->v_full[sv], blk_bytes);
        load(dv, &tm_vn, &tm_vc, &bars->v_full[sv]);
        ++gv;
        continue;
      }
      // Partial block or bad pages: both operands through the private
      // barrier, then zero the rows without a valid key and publish.
      if ((g >= NSK && !wait_all(&bars->k_empty[sk], phk ^ 1u, abort_flag, pb.err)) ||
          (g >= NSV && !wait_all(&bars->v_empty[sv], phv ^ 1u, abort_flag, pb.err))) {
        ok = false;
        break;
      }
      ptx::mbar_arrive_expect_tx_elect(&bars->fix[0], 2 * blk_bytes);
      load(dk, &tm_kn, &tm_kc, &bars->fix[0]);
      load(dv, &tm_vn, &tm_vc, &bars->fix[0]);
      // the private barrier completes even when no copy was queued
      const bool fok = wait_all(&bars->fix[0], fix_phase, abort_flag, pb.err);
      fix_phase ^= 1u;
      if (!fok) {
        // copies may still be in flight: the drain below waits for them
        fix_pending = true;
        ok = false;
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
  }
  // every copy this warp queued must land before the CTA ends
  if (lane == 0) {
    if (uq > 0) ptx::mbar_wait(&bars->q_full, (uint32_t)((uq - 1) & 1));
    for (int k = gk - NSK < 0 ? 0 : gk - NSK; k < gk; ++k)
      ptx::mbar_wait(&bars->k_full[k % NSK], (uint32_t)((k / NSK) & 1));
    for (int k = gv - NSV < 0 ? 0 : gv - NSV; k < gv; ++k)
      ptx::mbar_wait(&bars->v_full[k % NSV], (uint32_t)((k / NSV) & 1));
    if (fix_pending) ptx::mbar_wait(&bars->fix[0], fix_phase ^ 1u);
  }
  __syncwarp();
}

// One producer warp per operand (IS_V: V, else Q and K): each ring is filled
// as soon as its own stages are released, so K runs a full ring ahead of
// the QKs whatever the V ring waits for.  Used for batches whose prefill work
// is mostly paged context, where the gathers are latency-bound.  Same block
// handling as produce_kv, with a private barrier per operand.
template <int D, bool IS_V>
__device__ __forceinline__ void produce(Bars2 *bars, volatile int *abort_flag, const Problem pb,
                                        const PrefillTile *tiles, int n_units, uint8_t *sQ, uint8_t *sOp,
                                        const CUtensorMap *tm_q, const CUtensorMap *tm_new,
                                        const CUtensorMap *tm_ctx) {
  using S = P2Shape<D>;
  constexpr int BM = S::BM, BN = S::BN, NS = IS_V ? S::NSV : S::NSK;
  uint64_t *full = IS_V ? bars->v_full : bars->k_full;
  uint64_t *empty = IS_V ? bars->v_empty : bars->k_empty;
  uint64_t *fixb = &bars->fix[IS_V ? 1 : 0];
  const int lane = threadIdx.x & 31;
  const uint64_t once = ptx::l2_evict_first_policy();   // for the Q tiles (read once)
  const int br = pb.p < BN ? pb.p : BN;
  const int nseg = BN / br;
  uint32_t fix_phase = 0;
  int g = 0;            // blocks started so far (all units)
  int gp = 0;           // blocks whose copies were queued and published
  bool fix_pending = false;
  int uq = 0;           // units started
  bool ok = true;
  PrefillTile next = load_tile(tiles, unit_of(0), n_units, pb.hq);
  for (int r = 0, u = unit_of(0); ok && u < n_units; u = unit_of(++r), ++uq) {
    const Unit w = make_unit<BM, BN>(next, u, pb);
    next = load_tile(tiles, unit_of(r + 1), n_units, pb.hq);
    if (w.tile.rows == 0) break;   // end of a device-planned tile list
    const int32_t *pt_row = pb.page_table + (size_t)w.tile.seq * pb.max_pages;
    if (!IS_V) {
      // Q of both tiles, once the previous unit's QK MMAs are done with sQ
      if (uq > 0 && !wait_all(&bars->q_empty, (uint32_t)((uq - 1) & 1), abort_flag, pb.err)) break;
      ptx::mbar_arrive_expect_tx_elect(&bars->q_full, (w.rows_t[1] > 0 ? 2 : 1) * S::kQBytes);
      for (int t = 0; t < 2; ++t) {
        if (w.rows_t[t] == 0) continue;
        for (int hh = 0; hh < S::kHalves; ++hh)
          ptx::tma_load_3d_hint_elect(sQ + t * S::kQBytes + hh * BM * 128, tm_q, &bars->q_full, hh * 64, w.h,
                                      w.tile.q_start + w.r0 + t * BM, once);
      }
    }
    // page of this lane's segment of context block j (-1: no such segment)
    auto page_of = [&](int j) -> int {
      const int sp = j * BN + lane * br;
      return (j < w.n_ctx && lane < nseg && sp < w.c) ? pt_row[sp / pb.p] : -1;
    };
    int page_next = page_of(0);
    for (int j = 0; j < w.nb; ++j, ++g) {
      const int page = page_next;
      if (j + 1 < w.nb) page_next = page_of(j + 1);
      const int s = g % NS;
      const uint32_t ph = (uint32_t)((g / NS) & 1);
      uint8_t *dst = sOp + s * S::kKVBytes;
      const bool ctx = j < w.n_ctx;
      const int pos0 = ctx ? j * BN : (j - w.n_ctx) * BN;
      const int valid = min(BN, (ctx ? w.c : w.tile.q_len) - pos0);
      bool seg_loaded = false, seg_bad = false;
      if (ctx && lane < nseg && pos0 + lane * br < w.c) {
        if (page < 0 || page >= pb.num_pages) {
          seg_bad = true;
          if (!IS_V) atomicOr(pb.err, RPA_DEV_BAD_PAGE);
        } else {
          seg_loaded = true;
        }
      }
      const unsigned loaded_mask = __ballot_sync(0xffffffffu, seg_loaded);
      const bool fix = valid < BN || __any_sync(0xffffffffu, seg_bad);
      const uint32_t seg_bytes = (uint32_t)(S::kHalves * br * 128);
      const uint32_t blk_bytes = ctx ? (uint32_t)__popc(loaded_mask) * seg_bytes : (uint32_t)S::kKVBytes;
      if (g >= NS && !wait_all(&empty[s], ph ^ 1u, abort_flag, pb.err)) {
        ok = false;
        break;
      }
      uint64_t *bar = fix ? fixb : &full[s];
      ptx::mbar_arrive_expect_tx_elect(bar, blk_bytes);
      if (!ctx) {
        const int row = w.tile.q_start + pos0;
        for (int hh = 0; hh < S::kHalves; ++hh)
          ptx::tma_load_3d_elect(dst + hh * BN * 128, tm_new, bar, hh * 64, w.hk, row);
      } else {
        // each lane queues the copies of its own page segment
        if ((loaded_mask >> lane) & 1u) {
          const int row = page * pb.p + ((pos0 + lane * br) % pb.p);
          for (int hh = 0; hh < S::kHalves; ++hh)
            ptx::tma_load_3d(dst + hh * BN * 128 + lane * br * 128, tm_ctx, bar, hh * 64, w.hk, row);
        }
        __syncwarp();
      }
      if (fix) {
        // the private barrier completes even when no copy was queued
        const bool fok = wait_all(fixb, fix_phase, abort_flag, pb.err);
        fix_phase ^= 1u;
        if (!fok) {
          fix_pending = true;   // copies may still be in flight: drained below
          ok = false;
          break;
        }
        for (int rr = lane; rr < BN; rr += 32) {
          const bool bad_row = rr >= valid || (ctx && !((loaded_mask >> (rr / br)) & 1u));
          if (!bad_row) continue;
          for (int hh = 0; hh < S::kHalves; ++hh) {
            uint4 *pz = reinterpret_cast<uint4 *>(dst + hh * BN * 128 + rr * 128);
#pragma unroll
            for (int q = 0; q < 8; ++q) pz[q] = make_uint4(0, 0, 0, 0);
          }
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        ptx::mbar_arrive_elect(&full[s]);
      }
      ++gp;
    }
  }
  // every copy this warp queued must land before the CTA ends
  if (lane == 0) {
    if (!IS_V && uq > 0) ptx::mbar_wait(&bars->q_full, (uint32_t)((uq - 1) & 1));
    for (int k = gp - NS < 0 ? 0 : gp - NS; k < gp; ++k) ptx::mbar_wait(&full[k % NS], (uint32_t)((k / NS) & 1));
    if (fix_pending) ptx::mbar_wait(fixb, fix_phase ^ 1u);
  }
  __syncwarp();
}

// The fused cache update: threads [0, n) of the cache-writer warps copy this
// CTA's share of the new K/V rows (one of the G query heads of each KV head
// takes each row of an item) from k_new / v_new into their page slots.
template <int D>
__device__ __forceinline__ void cache_update(const Problem pb, const PrefillTile *tiles, int n_units, int wt,
                                             int n) {
  using S = P2Shape<D>;
  constexpr int BM = S::BM, BN = S::BN;
  if (!kCacheWrite) return;
  const int G = pb.hq / pb.hkv;
  const int chunks = D / 8;
  const __nv_bfloat16 *kn = reinterpret_cast<const __nv_bfloat16 *>(pb.k_new);
  const __nv_bfloat16 *vn = reinterpret_cast<const __nv_bfloat16 *>(pb.v_new);
  __nv_bfloat16 *kc = reinterpret_cast<__nv_bfloat16 *>(pb.k_cache);
  __nv_bfloat16 *vc = reinterpret_cast<__nv_bfloat16 *>(pb.v_cache);
  const uint64_t once = ptx::l2_evict_first_policy();
  PrefillTile next = load_tile(tiles, unit_of(0), n_units, pb.hq);
  for (int r = 0, u = unit_of(0); u < n_units; u = unit_of(++r)) {
    const Unit w = make_unit<BM, BN>(next, u, pb);
    next = load_tile(tiles, unit_of(r + 1), n_units, pb.hq);
    if (w.tile.rows == 0) break;   // end of a device-planned tile list
    const int32_t *pt_row = pb.page_table + (size_t)w.tile.seq * pb.max_pages;
    const int gidx = w.h % G;
    const int ra = (gidx * w.tile.rows) / G, rb = ((gidx + 1) * w.tile.rows) / G;
    for (int idx = wt; idx < (rb - ra) * chunks; idx += n) {
      const int i = w.r0 + ra + idx / chunks;   // new-token index
      const int ch = idx % chunks;
      const int pos = w.c + i;
      const int pg = pt_row[pos / pb.p];
      if (pg < 0 || pg >= pb.num_pages) {
        if (ch == 0) atomicOr(pb.err, RPA_DEV_BAD_PAGE);
        continue;
      }
      const size_t src = ((size_t)(w.tile.q_start + i) * pb.hkv + w.hk) * D + ch * 8;
      const size_t dst = (((size_t)pg * pb.p + pos % pb.p) * pb.hkv + w.hk) * D + ch * 8;
      // written once and not read again by this launch: first out of L2,
      // ahead of the K/V blocks that other query heads still read
      ptx::st_global_hint(kc + dst, *reinterpret_cast<const uint4 *>(kn + src), once);
      ptx::st_global_hint(vc + dst, *reinterpret_cast<const uint4 *>(vn + src), once);
    }
  }
}

// Persistent: each CTA walks its units in the order of unit_of() over the
// list of (item, query head) units; items are sorted heaviest first on the
// host and the heads of one item are consecutive (their K/V blocks are
// shared in L2).
// Every barrier parity runs on counters that span units, so the producer
// loads the next unit's Q and K/V while the current one finishes and the MMA
// warp starts the next unit while the softmax warps are still storing O.
// split: V gets a producer warp of its own (warp 10) and the cache update
// one warp (11); otherwise warp 8 loads K and V and warps 10-11 update the
// cache.  A device-planned call passes the capacity's unit count; the
// planner ends the tile list with empty tiles and chooses split.
template <int D>
__global__ void __launch_bounds__(384, 1)
    prefill2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                    const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kn,
                    const __grid_constant__ CUtensorMap tm_vn, const Problem pb,
                    const PrefillTile *__restrict__ tiles, int n_units, int split, float scale_log2) {
  using S = P2Shape<D>;
  constexpr int BM = S::BM, BN = S::BN, NSK = S::NSK, NSV = S::NSV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = base;                              // tile t at sQ + t * kQBytes
  uint8_t *sK = sQ + 2 * S::kQBytes;
  uint8_t *sV = sK + NSK * S::kKVBytes;
  Bars2 *bars = reinterpret_cast<Bars2 *>(base + S::kData);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (pb.dev_counts != nullptr) {
    // capacity-sized grid: CTAs without a unit leave before any set-up
    if ((int)blockIdx.x >= pb.dev_counts[kCntPrefill] * pb.hq) return;
    split = pb.dev_counts[kCntPrefillSplit];
  }

  if (tid == 0) {
    ptx::mbar_init(&bars->q_full, 1);
    ptx::mbar_init(&bars->q_empty, 1);
    for (int i = 0; i < NSK; ++i) {
      ptx::mbar_init(&bars->k_full[i], 1);
      ptx::mbar_init(&bars->k_empty[i], 1);
    }
    for (int i = 0; i < NSV; ++i) {
      ptx::mbar_init(&bars->v_full[i], 1);
      ptx::mbar_init(&bars->v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->s_full[i], 1);
      ptx::mbar_init(&bars->p_full[i], 128);
      ptx::mbar_init(&bars->p_half[i], 128);
      ptx::mbar_init(&bars->pv_done[i], 1);
      ptx::mbar_init(&bars->o_free[i], 128);
    }
    ptx::mbar_init(&bars->fix[0], 1);
    ptx::mbar_init(&bars->fix[1], 1);
    ptx::mbar_init(&bars->drain, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 9) {
    ptx::tmem_alloc(tmem_slot, S::kTmemCols);
    ptx::tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
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

  if (warp >= 8) {
    setmaxnreg_dec96();
    if (warp == 8) {
      if (split)
        produce<D, false>(bars, abort_flag, pb, tiles, n_units, sQ, sK, &tm_q, &tm_kn, &tm_kc);
      else
        produce_kv<D>(bars, abort_flag, pb, tiles, n_units, sQ, sK, sV, &tm_q, &tm_kc, &tm_vc, &tm_kn, &tm_vn);
    } else if (warp == 9) {
      // --------------------------------------------------------------- MMA
      mma_loop<D>(bars, abort_flag, pb, tiles, n_units, tmem, ptx::smem_u32(sQ), ptx::smem_u32(sK),
                  ptx::smem_u32(sV));
    } else if (split && warp == 10) {
      produce<D, true>(bars, abort_flag, pb, tiles, n_units, sQ, sV, &tm_q, &tm_vn, &tm_vc);
    } else {
      // fused cache update: warps 10-11, or warp 11 when warp 10 loads V
      cache_update<D>(pb, tiles, n_units, split ? lane : tid - 320, split ? 32 : 64);
    }
  } else {
    // ----------------------------------------------------------- softmax
    setmaxnreg_inc200();
    const int t = warp >> 2;                     // tile
    const int row = tid & 127;                   // TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t tS = lane_base + (uint32_t)(t * 128);
    const uint32_t tO = lane_base + S::kColO + (uint32_t)(t * D);
    int gt = 0;                                  // blocks of this tile consumed so far
    int ep = 0;                                  // units in which this tile had rows
    bool ok = true;
    PrefillTile next = load_tile(tiles, unit_of(0), n_units, pb.hq);
    for (int r = 0, u = unit_of(0); ok && u < n_units; u = unit_of(++r)) {
      const Unit w = make_unit<BM, BN>(next, u, pb);
      next = load_tile(tiles, unit_of(r + 1), n_units, pb.hq);
      if (w.tile.rows == 0) break;   // end of a device-planned tile list
      // tile-uniform selects keep the unit in registers (no local memory)
      const int n = t ? w.n_t[1] : w.n_t[0];
      const int rows_mine = t ? w.rows_t[1] : w.rows_t[0];
      const int rn = w.r0 + t * BM + row;        // new-token index of this row
      float m = -INFINITY, l = 0.f, lr = 0.f;   // lr: the normaliser of O (below)
      for (int j = 0; j < n; ++j) {
        if (!__all_sync(0xffffffffu,
                        wait_bar2(&bars->s_full[t], (uint32_t)((gt + j) & 1), abort_flag, pb.err))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        float x[BN];
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc)
          ptx::tmem_ld32(tS + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&x[cc * 32]));
        ptx::tmem_ld_wait();
        int lim;
        if (j < w.n_ctx) {
          lim = min(BN, w.c - j * BN);
        } else {
          const int kn0 = (j - w.n_ctx) * BN;
          const int end = pb.causal ? min(w.tile.q_len, rn + 1) : w.tile.q_len;
          lim = max(0, min(BN, end - kn0));
        }
        const bool masked = __any_sync(0xffffffffu, lim < BN);
        if (masked) {
#pragma unroll
          for (int i = 0; i < BN; ++i) x[i] = i < lim ? x[i] : -INFINITY;
        }
        // row max of the raw scores: 4 chains of 3-input max
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
        const bool need = m != -INFINITY && m_new > m + kRescaleThreshold;
        float alpha = 1.f;
        if (__any_sync(0xffffffffu, need)) {
          // PV(t, j-1) has completed: s_full(t, j) was committed after QK(t, j),
          // which was issued after PV(t, j-1).
          alpha = (m_new == m) ? 1.f : ptx::ex2(m - m_new);
          if (j > 0) {
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
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
        uint64_t sp2[4] = {0, 0, 0, 0};   // packed partial sums (+0.0f pairs)
        uint32_t pk[BN / 2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
          for (int i = hf * (BN / 2); i < (hf + 1) * (BN / 2); i += 2) {
            float a0, a1;
            ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(x[i], x[i + 1]), scale2, negm2), a0, a1);
            const uint64_t pp = ptx::f2_pack(ptx::ex2(a0), ptx::ex2(a1));
            sp2[(i >> 1) & 3] = ptx::f2_add(sp2[(i >> 1) & 3], pp);
            float p0, p1;
            ptx::f2_unpack(pp, p0, p1);
            pk[i >> 1] = ptx::pack_bf16(p0, p1);
          }
          // P of keys [64 hf, 64 hf + 64) as bf16 into S's columns [32 hf, 32 hf + 32)
          ptx::tmem_st32(tS + hf * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[hf * 32]));
          if (hf == 0) {
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            ptx::mbar_arrive(&bars->p_half[t]);
          }
        }
        float sp[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) ptx::f2_unpack(sp2[k], sp[2 * k], sp[2 * k + 1]);
        const float sum = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
        // The PV MMA takes P rounded to bf16.  Under the lazy rescale the
        // block's largest weight can be up to 2^8 (not exactly 1), and its
        // rounding (relative 2^-9) moves O by up to 2^-9 |V| when one key
        // dominates the row.  lr, the normaliser of O, therefore counts that
        // weight as rounded, so that its rounding cancels in O / lr; the
        // other weights keep the error of a kernel whose max weight is 1.
        // l keeps the exact fp32 sum, for lse.
        const float pmax = ptx::ex2(fmaf(mraw, scale_log2, neg_m));   // as the loop computed it
        l = l * alpha + sum;
        lr = lr * alpha + (sum - (pmax - ptx::round_bf16(pmax)));
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->p_full[t]);
      }
      if (!ok || n == 0) continue;
      gt += n;
      // one pv_done phase per unit of this tile (committed after its last PV)
      if (!__all_sync(0xffffffffu, wait_bar2(&bars->pv_done[t], (uint32_t)(ep & 1), abort_flag, pb.err))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const float inv = 1.f / lr;
      const bool store = row < rows_mine;
      __nv_bfloat16 *out =
          reinterpret_cast<__nv_bfloat16 *>(pb.out) + ((size_t)(w.tile.q_start + rn) * pb.hq + w.h) * D;
      // all of O_t into registers with one wait, then O_t is free for the
      // next unit's first PV while the rows are stored
      uint32_t ov[D];
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) ptx::tmem_ld32(tO + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[cc * 32]));
      ptx::tmem_ld_wait();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->o_free[t]);
      if (store) {
        const uint64_t once = ptx::l2_evict_first_policy();   // written once: first out of L2
#pragma unroll
        for (int cc = 0; cc < D / 8; ++cc) {
          uint32_t o2[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            o2[i] = ptx::pack_bf16(__uint_as_float(ov[cc * 8 + 2 * i]) * inv, __uint_as_float(ov[cc * 8 + 2 * i + 1]) * inv);
          ptx::st_global_hint(reinterpret_cast<uint4 *>(out) + cc, make_uint4(o2[0], o2[1], o2[2], o2[3]), once);
        }
      }
      ++ep;
      if (store && pb.lse != nullptr) pb.lse[(size_t)(w.tile.q_start + rn) * pb.hq + w.h] = (m + log2f(l)) * kLn2;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 9) ptx::tmem_dealloc(tmem, S::kTmemCols);
}

template <int D>
cudaError_t launch_t(const Problem &pb, const PrefillTile *tiles, int n_tiles, int max_ctas, bool split,
                     cudaStream_t stream) {
  using S = P2Shape<D>;
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
  auto kern = prefill2_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem);
  if (e != cudaSuccess) return e;
  const int n_units = n_tiles * pb.hq;
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      sms = 148;
  }
  int grid = n_units < sms ? n_units : sms;
  if (max_ctas > 0 && grid > max_ctas) grid = max_ctas;
  kern<<<grid, 384, S::kSmem, stream>>>(tq, tkc, tvc, tkn, tvn, pb, tiles, n_units, split ? 1 : 0,
                                        pb.scale * kLog2e);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill2(const Problem &pb, const PrefillTile *tiles, int n_tiles, int max_ctas, bool split,
                            cudaStream_t stream) {
  if (n_tiles <= 0) return cudaSuccess;
  switch (pb.d) {
    case 64: return launch_t<64>(pb, tiles, n_tiles, max_ctas, split, stream);
    case 128: return launch_t<128>(pb, tiles, n_tiles, max_ctas, split, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rpa
