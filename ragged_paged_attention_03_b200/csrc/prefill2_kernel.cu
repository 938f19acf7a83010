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
//   warp 9                   TMEM owner, single-thread tcgen05.mma issue
//   warps 10-11              fused cache update: this CTA's share of the new
//                            K/V rows copied into their page slots
//
// TMEM (512 columns): S/P of tile 0 | S/P of tile 1 | O of tile 0 | O of tile 1.
// P overwrites its tile's S as bf16 and is the A operand of O += P V.  MMA
// issue order per key block j: PV(0,j), QK(0,j+1), PV(1,j), QK(1,j+1).
//
// exp2 on the multi-function unit is the softmax bottleneck on this part, so
// a quarter of the exponentials are computed on the FMA pipe instead: round
// x to the nearest integer n, f = x - n in [-1/2, 1/2], 2^f by a degree-3
// polynomial fitted for minimax relative error (max 7.5e-5, far below the
// bf16 rounding of P), and 2^n added into the exponent field.
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
  static constexpr int NS = D == 64 ? 3 : 2;
  static constexpr int kHalves = D / 64;
  static constexpr int kQBytes = kHalves * BM * 128;
  static constexpr int kKVBytes = kHalves * BN * 128;
  static constexpr int kData = 2 * kQBytes + 2 * NS * kKVBytes;
  static constexpr int kSmem = 1024 + kData + 512;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 256;   // O of tile t at kColO + t * D
};

struct Bars2 {
  uint64_t q_full, q_empty;
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint64_t s_full[2], p_full[2], pv_done[2], o_free[2];
  uint64_t fix, drain;
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

// 2^x for x <= ~8 on the FMA pipe (see the file comment).
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -125.0f);                   // keeps n >= -125: 2^n stays a normal number
  const float r = x + 12582912.0f;          // 1.5 * 2^23: x rounded to nearest in the low bits
  const float n = r - 12582912.0f;
  const float f = x - n;
  float p = fmaf(0.0551709607f, f, 0.242609662f);
  p = fmaf(p, f, 0.693260965f);
  p = fmaf(p, f, 0.999928165f);
  const int ni = __float_as_int(r) - 0x4B400000;
  return __int_as_float(__float_as_int(p) + (ni << 23));
}

// The same on a packed pair: (x0, x1) -> (2^x0, 2^x1), with x already
// clamped to >= -125.
__device__ __forceinline__ uint64_t exp2_fma2(float x0, float x1) {
  const uint64_t x = ptx::f2_pack(x0, x1);
  const uint64_t magic = ptx::f2_pack(12582912.0f, 12582912.0f);
  const uint64_t neg_magic = ptx::f2_pack(-12582912.0f, -12582912.0f);
  const uint64_t r = ptx::f2_add(x, magic);
  const uint64_t n = ptx::f2_add(r, neg_magic);
  const uint64_t f = ptx::f2_fma(n, ptx::f2_pack(-1.0f, -1.0f), x);
  uint64_t p = ptx::f2_fma(ptx::f2_pack(0.0551709607f, 0.0551709607f), f, ptx::f2_pack(0.242609662f, 0.242609662f));
  p = ptx::f2_fma(p, f, ptx::f2_pack(0.693260965f, 0.693260965f));
  p = ptx::f2_fma(p, f, ptx::f2_pack(0.999928165f, 0.999928165f));
  float r0, r1, p0, p1;
  ptx::f2_unpack(r, r0, r1);
  ptx::f2_unpack(p, p0, p1);
  const int n0 = __float_as_int(r0) - 0x4B400000, n1 = __float_as_int(r1) - 0x4B400000;
  return ptx::f2_pack(__int_as_float(__float_as_int(p0) + (n0 << 23)),
                      __int_as_float(__float_as_int(p1) + (n1 << 23)));
}

__device__ __forceinline__ void setmaxnreg_inc200() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 200;" ::: "memory");
}
__device__ __forceinline__ void setmaxnreg_dec96() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 96;" ::: "memory");
}

// Geometry of one work unit (a 256-row item of one sequence, one query head).
struct Unit {
  PrefillTile tile;
  int h, hk, c, r0, n_ctx, nb;
  int rows_t[2], n_t[2];
};

template <int BM, int BN>
__device__ __forceinline__ Unit make_unit(const PrefillTile *tiles, int u, const Problem &pb) {
  Unit w;
  w.tile = tiles[u / pb.hq];
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

// Persistent: CTA b handles units b, b + gridDim.x, ... of the list of
// (item, query head) units; items are sorted heaviest first on the host and
// the heads of one item are consecutive (their K/V blocks are shared in L2).
// Every barrier parity runs on counters that span units, so the producer
// loads the next unit's Q and K/V while the current one finishes and the MMA
// warp starts the next unit while the softmax warps are still storing O.
template <int D>
__global__ void __launch_bounds__(384, 1)
    prefill2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                    const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kn,
                    const __grid_constant__ CUtensorMap tm_vn, const Problem pb,
                    const PrefillTile *__restrict__ tiles, int n_units, float scale_log2) {
  using S = P2Shape<D>;
  constexpr int BM = S::BM, BN = S::BN, NS = S::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = base;                              // tile t at sQ + t * kQBytes
  uint8_t *sK = sQ + 2 * S::kQBytes;
  uint8_t *sV = sK + NS * S::kKVBytes;
  Bars2 *bars = reinterpret_cast<Bars2 *>(base + S::kData);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = pb.hq / pb.hkv;

  if (tid == 0) {
    ptx::mbar_init(&bars->q_full, 1);
    ptx::mbar_init(&bars->q_empty, 1);
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(&bars->k_full[i], 1);
      ptx::mbar_init(&bars->k_empty[i], 1);
      ptx::mbar_init(&bars->v_full[i], 1);
      ptx::mbar_init(&bars->v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->s_full[i], 1);
      ptx::mbar_init(&bars->p_full[i], 128);
      ptx::mbar_init(&bars->pv_done[i], 1);
      ptx::mbar_init(&bars->o_free[i], 128);
    }
    ptx::mbar_init(&bars->fix, 1);
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
      // ---------------------------------------------------------- producer
      const int br = pb.p < BN ? pb.p : BN;
      const int nseg = BN / br;
      uint32_t fix_phase = 0;
      int g = 0;            // K/V blocks queued so far (all units)
      int uq = 0;           // units started
      bool ok = true;
      for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++uq) {
        const Unit w = make_unit<BM, BN>(tiles, u, pb);
        const int32_t *pt_row = pb.page_table + (size_t)w.tile.seq * pb.max_pages;
        // Q of both tiles, once the previous unit's QK MMAs are done with sQ
        if (uq > 0 && !wait_bar2(&bars->q_empty, (uint32_t)((uq - 1) & 1), abort_flag, pb.err)) break;
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(&bars->q_full, (w.rows_t[1] > 0 ? 2 : 1) * S::kQBytes);
          for (int t = 0; t < 2; ++t) {
            if (w.rows_t[t] == 0) continue;
            for (int hh = 0; hh < S::kHalves; ++hh)
              ptx::tma_load_3d(sQ + t * S::kQBytes + hh * BM * 128, &tm_q, &bars->q_full, hh * 64, w.h,
                               w.tile.q_start + w.r0 + t * BM);
          }
        }
        for (int j = 0; j < w.nb; ++j, ++g) {
          const int s = g % NS;
          const uint32_t ph = (uint32_t)((g / NS) & 1);
          uint8_t *dk = sK + s * S::kKVBytes;
          uint8_t *dv = sV + s * S::kKVBytes;
          const bool ctx = j < w.n_ctx;
          const int pos0 = ctx ? j * BN : (j - w.n_ctx) * BN;
          const int valid = min(BN, (ctx ? w.c : w.tile.q_len) - pos0);
          int page = -1;
          bool seg_loaded = false, seg_bad = false;
          if (ctx && lane < nseg) {
            const int sp = pos0 + lane * br;
            if (sp < w.c) {
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
          if (g >= NS) {
            if (!wait_bar2(&bars->k_empty[s], ph ^ 1u, abort_flag, pb.err) ||
                !wait_bar2(&bars->v_empty[s], ph ^ 1u, abort_flag, pb.err)) {
              ok = false;
              break;
            }
          }
          uint64_t *kb = fix ? &bars->fix : &bars->k_full[s];
          uint64_t *vb = fix ? &bars->fix : &bars->v_full[s];
          if (lane == 0) {
            if (fix) {
              ptx::mbar_arrive_expect_tx(&bars->fix, 2 * blk_bytes);
            } else {
              ptx::mbar_arrive_expect_tx(&bars->k_full[s], blk_bytes);
              ptx::mbar_arrive_expect_tx(&bars->v_full[s], blk_bytes);
            }
            if (!ctx) {
              const int row = w.tile.q_start + pos0;
              for (int hh = 0; hh < S::kHalves; ++hh) {
                ptx::tma_load_3d(dk + hh * BN * 128, &tm_kn, kb, hh * 64, w.hk, row);
                ptx::tma_load_3d(dv + hh * BN * 128, &tm_vn, vb, hh * 64, w.hk, row);
              }
            }
          }
          if (ctx) {
            for (int sg = 0; sg < nseg; ++sg) {
              const int pg = __shfl_sync(0xffffffffu, page, sg);
              if (lane != 0 || !((loaded_mask >> sg) & 1u)) continue;
              const int sp = pos0 + sg * br;
              const int row = pg * pb.p + (sp % pb.p);
              for (int hh = 0; hh < S::kHalves; ++hh) {
                ptx::tma_load_3d(dk + hh * BN * 128 + sg * br * 128, &tm_kc, kb, hh * 64, w.hk, row);
                ptx::tma_load_3d(dv + hh * BN * 128 + sg * br * 128, &tm_vc, vb, hh * 64, w.hk, row);
              }
            }
          }
          if (fix) {
            // wait for this block's copies (the private barrier completes
            // even with none), zero the rows without a valid key, publish
            const bool fok = wait_bar2(&bars->fix, fix_phase, abort_flag, pb.err);
            fix_phase ^= 1u;
            if (!fok) {
              ok = false;
              ++g;
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
            if (lane == 0) {
              ptx::mbar_arrive(&bars->k_full[s]);
              ptx::mbar_arrive(&bars->v_full[s]);
            }
          }
        }
      }
      // every copy this warp queued must land before the CTA ends
      if (lane == 0) {
        if (uq > 0) ptx::mbar_wait(&bars->q_full, (uint32_t)((uq - 1) & 1));
        for (int k = g - NS < 0 ? 0 : g - NS; k < g; ++k) {
          ptx::mbar_wait(&bars->k_full[k % NS], (uint32_t)((k / NS) & 1));
          ptx::mbar_wait(&bars->v_full[k % NS], (uint32_t)((k / NS) & 1));
        }
      }
      __syncwarp();
    } else if (warp == 9) {
      // --------------------------------------------------------------- MMA
      if (lane == 0) {
        const uint32_t tS[2] = {tmem, tmem + 128};
        const uint32_t tO[2] = {tmem + S::kColO, tmem + S::kColO + D};
        constexpr uint32_t idesc_qk = ptx::umma_idesc_bf16(128, BN, false);
        constexpr uint32_t idesc_pv = ptx::umma_idesc_bf16(128, D, true);
        const uint32_t q_addr = ptx::smem_u32(sQ);
        const uint32_t k_addr = ptx::smem_u32(sK);
        const uint32_t v_addr = ptx::smem_u32(sV);
        int g0 = 0;              // first global block index of the unit
        int gt[2] = {0, 0};      // blocks of each tile consumed so far
        int ep[2] = {0, 0};      // units in which each tile was active
        bool ok = true;
        // Descriptors of the stage-0 / tile-0 operands; the start-address
        // field is the low 14 bits (address / 16), so other stages, tiles,
        // k-steps and column tiles are reached by adding (offset / 16).
        const uint64_t dq0 = ptx::umma_desc_sw128(q_addr, 16, 1024);
        const uint64_t dk0 = ptx::umma_desc_sw128(k_addr, 16, 1024);
        const uint64_t dv0 = ptx::umma_desc_sw128(v_addr, BN * 128, 1024);
        auto qk = [&](int t, int gblk) -> bool {
          const int s = gblk % NS;
          if (!wait_bar2(&bars->k_full[s], (uint32_t)((gblk / NS) & 1), abort_flag, pb.err)) return false;
          ptx::tc_fence_after();
          const uint64_t dq = dq0 + (uint64_t)((t * S::kQBytes) >> 4);
          const uint64_t dk = dk0 + (uint64_t)((s * S::kKVBytes) >> 4);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = ((ks >> 2) * BM * 128 + (ks & 3) * 32) >> 4;
            const uint32_t offk = ((ks >> 2) * BN * 128 + (ks & 3) * 32) >> 4;
            ptx::umma_ss(tS[t], dq + off, dk + offk, idesc_qk, ks > 0 ? 1u : 0u);
          }
          ptx::umma_commit(&bars->s_full[t]);
          return true;
        };
        auto pv = [&](int t, int gblk, int tblk, bool first) -> bool {
          const int s = gblk % NS;
          if (!wait_bar2(&bars->p_full[t], (uint32_t)(tblk & 1), abort_flag, pb.err)) return false;
          if (!wait_bar2(&bars->v_full[s], (uint32_t)((gblk / NS) & 1), abort_flag, pb.err)) return false;
          ptx::tc_fence_after();
          const uint64_t dv = dv0 + (uint64_t)((s * S::kKVBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            ptx::umma_ts(tO[t], tS[t] + kk * 8, dv + (uint64_t)((kk * 16 * 128) >> 4), idesc_pv,
                         (!first || kk > 0) ? 1u : 0u);
          ptx::umma_commit(&bars->pv_done[t]);
          return true;
        };
        int uq = 0;
        for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++uq) {
          const Unit w = make_unit<BM, BN>(tiles, u, pb);
          ok = wait_bar2(&bars->q_full, (uint32_t)(uq & 1), abort_flag, pb.err);
          // first QK of each tile: its S/P buffer must have been read by the
          // previous unit's last PV
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (!ok || w.n_t[t] == 0) continue;
            if (gt[t] > 0) ok = wait_bar2(&bars->pv_done[t], (uint32_t)((gt[t] - 1) & 1), abort_flag, pb.err);
            if (ok) ok = qk(t, g0);
          }
          if (ok) ptx::umma_commit(&bars->k_empty[g0 % NS]);
          if (ok && w.nb == 1) ptx::umma_commit(&bars->q_empty);
          for (int j = 0; ok && j < w.nb; ++j) {
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (ok && j < w.n_t[t]) {
                // O of tile t is overwritten by the unit's first PV: the
                // softmax warps must have read the previous unit's O
                if (j == 0 && ep[t] > 0)
                  ok = wait_bar2(&bars->o_free[t], (uint32_t)((ep[t] - 1) & 1), abort_flag, pb.err);
                if (ok) ok = pv(t, g0 + j, gt[t] + j, j == 0);
              }
              if (ok && j + 1 < w.n_t[t]) {
                ok = wait_bar2(&bars->pv_done[t], (uint32_t)((gt[t] + j) & 1), abort_flag, pb.err);
                if (ok) ok = qk(t, g0 + j + 1);
              }
            }
            if (ok) ptx::umma_commit(&bars->v_empty[(g0 + j) % NS]);
            if (ok && j + 1 < w.nb) ptx::umma_commit(&bars->k_empty[(g0 + j + 1) % NS]);
            if (ok && j + 2 == w.nb) ptx::umma_commit(&bars->q_empty);   // last QK of the unit issued
          }
          g0 += w.nb;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            gt[t] += w.n_t[t];
            ep[t] += w.n_t[t] > 0 ? 1 : 0;
          }
        }
        ptx::umma_commit(&bars->drain);
        ptx::mbar_wait(&bars->drain, 0);
      }
      __syncwarp();
    } else {
      // ------------------------------------------ fused cache update (64 thr)
      const int chunks = D / 8;
      const int wt = tid - 320;
      const __nv_bfloat16 *kn = reinterpret_cast<const __nv_bfloat16 *>(pb.k_new);
      const __nv_bfloat16 *vn = reinterpret_cast<const __nv_bfloat16 *>(pb.v_new);
      __nv_bfloat16 *kc = reinterpret_cast<__nv_bfloat16 *>(pb.k_cache);
      __nv_bfloat16 *vc = reinterpret_cast<__nv_bfloat16 *>(pb.v_cache);
      for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const Unit w = make_unit<BM, BN>(tiles, u, pb);
        const int32_t *pt_row = pb.page_table + (size_t)w.tile.seq * pb.max_pages;
        const int gidx = w.h % G;
        const int ra = (gidx * w.tile.rows) / G, rb = ((gidx + 1) * w.tile.rows) / G;
        for (int idx = wt; idx < (rb - ra) * chunks; idx += 64) {
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
          *reinterpret_cast<uint4 *>(kc + dst) = *reinterpret_cast<const uint4 *>(kn + src);
          *reinterpret_cast<uint4 *>(vc + dst) = *reinterpret_cast<const uint4 *>(vn + src);
        }
      }
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
    bool ok = true;
    for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
      const Unit w = make_unit<BM, BN>(tiles, u, pb);
      const int n = w.n_t[t];
      const int rn = w.r0 + t * BM + row;        // new-token index of this row
      float m = -INFINITY, l = 0.f;
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
        const float mx = ptx::fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3])) * scale_log2;
        const float m_new = fmaxf(m, mx);
        const bool need = m != -INFINITY && m_new > m + kRescaleThreshold;
        float alpha = 1.f;
        if (__any_sync(0xffffffffu, need)) {
          // PV(t, j-1) has completed: QK(t, j) was issued only after it.
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
        for (int i = 0; i < BN; i += 2) {
          float a0, a1;
          ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(x[i], x[i + 1]), scale2, negm2), a0, a1);
          uint64_t pp;
          if ((i & 7) == 6) {          // a quarter of the exponentials on the FMA pipe
            pp = exp2_fma2(fmaxf(a0, -125.0f), fmaxf(a1, -125.0f));
            if (masked) {
              float p0, p1;
              ptx::f2_unpack(pp, p0, p1);
              pp = ptx::f2_pack(i < lim ? p0 : 0.f, i + 1 < lim ? p1 : 0.f);
            }
          } else {
            pp = ptx::f2_pack(ptx::ex2(a0), ptx::ex2(a1));
          }
          sp2[(i >> 1) & 3] = ptx::f2_add(sp2[(i >> 1) & 3], pp);
          float p0, p1;
          ptx::f2_unpack(pp, p0, p1);
          pk[i >> 1] = ptx::pack_bf16(p0, p1);
        }
#pragma unroll
        for (int cc = 0; cc < BN / 64; ++cc)
          ptx::tmem_st32(tS + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[cc * 32]));
        float sp[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) ptx::f2_unpack(sp2[k], sp[2 * k], sp[2 * k + 1]);
        const float sum = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
        l = l * alpha + sum;
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->p_full[t]);
      }
      if (!ok || n == 0) continue;
      gt += n;
      if (!__all_sync(0xffffffffu, wait_bar2(&bars->pv_done[t], (uint32_t)((gt - 1) & 1), abort_flag, pb.err))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const float inv = 1.f / l;
      const bool store = row < w.rows_t[t];
      __nv_bfloat16 *out =
          reinterpret_cast<__nv_bfloat16 *>(pb.out) + ((size_t)(w.tile.q_start + rn) * pb.hq + w.h) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        ptx::tmem_ld32(tO + cc * 32, r);
        ptx::tmem_ld_wait();
        if (store) {
          uint32_t o2[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            o2[i] = ptx::pack_bf16(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
          uint4 *dst = reinterpret_cast<uint4 *>(out + cc * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(o2[4 * i], o2[4 * i + 1], o2[4 * i + 2], o2[4 * i + 3]);
        }
      }
      // O has been read: the next unit's first PV may overwrite it
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars->o_free[t]);
      if (store && pb.lse != nullptr) pb.lse[(size_t)(w.tile.q_start + rn) * pb.hq + w.h] = (m + log2f(l)) * kLn2;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 9) ptx::tmem_dealloc(tmem, S::kTmemCols);
}

template <int D>
cudaError_t launch_t(const Problem &pb, const PrefillTile *tiles, int n_tiles, cudaStream_t stream) {
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
  const int grid = n_units < sms ? n_units : sms;
  kern<<<grid, 384, S::kSmem, stream>>>(tq, tkc, tvc, tkn, tvn, pb, tiles, n_units, pb.scale * kLog2e);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill2(const Problem &pb, const PrefillTile *tiles, int n_tiles, cudaStream_t stream) {
  if (n_tiles <= 0) return cudaSuccess;
  switch (pb.d) {
    case 64: return launch_t<64>(pb, tiles, n_tiles, stream);
    case 128: return launch_t<128>(pb, tiles, n_tiles, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rpa
