// bsa_fwd_rows.cuh -- row-tile forward kernel (every block size).
//
// A tile is 128 query rows = R = 128 / block_size consecutive block rows of
// one (b, h).  The kernel walks the union of the tile's column lists in steps
// of 128 keys (128 / block_size blocks gathered into one shared-memory stage):
//
//   S = Q K_step^T            tcgen05.mma, M=128 queries, N=128 keys, K=d
//   P = 2^(S*scale*log2e - m) fp32 in registers, written back to TMEM as bf16
//   O += P V_step             tcgen05.mma with A = P read from TMEM, N=d
//
// A block row that does not hold a block of the step gets P = 0 there and its
// statistics skip it, so every row sums exactly over its own blocks ("Block
// Sparse Attention with Log-Linear Complexity", section 3.3); the exponentials
// of such blocks are not evaluated (membership is uniform over a warp).
//
// One persistent CTA per SM.  S is held in NS TMEM buffers and O in two, so
// the MMA issuer runs NS - 1 steps ahead of the softmax: while the softmax
// turns S(j) into P(j), the tensor core computes the next scores; then
// O += P(j) V(j) and S(j+NS).  A tile's first steps overlap the previous
// tile's epilogue the same way.  Roles (576 threads):
//   warps 0-15  softmax: warpgroup q takes keys 32q..32q+31 of every step for
//               all 128 rows (TMEM lane quadrant warp % 4) and O columns
//               [q d/4, (q+1) d/4) in the epilogue
//   warp 16     tile schedule, per-tile block bitmaps, TMA loads of Q, K, V
//   warp 17     tcgen05.mma issuer (and owner of the 512 TMEM columns)
// The four warps holding the same rows exchange their partial row maxima each
// step through shared memory (an mbarrier with bounded waits, not a hardware
// barrier, so that a warp giving up cannot leave the others waiting); their
// partial sums are added at the end of the tile.
//
// TMEM columns: S(j) in [128 (j mod NS), +128); warpgroup q writes P of its
// 32 keys over the first 16 of its own 32 score columns; O of tile t in
// [128 NS + d (t&1), +d).
//
// Work split (`schedule`): tiles whose estimated cost (longest row plus one
// step) exceeds half of a CTA's share -- the global rows of the local+global
// pattern -- are dealt out one per CTA first; the other tiles go out in
// round-robin rounds so that concurrent CTAs share K/V blocks in L2.
#pragma once

#include "bsa_common.cuh"

namespace bsa {
namespace rows {

constexpr int kSoftWG = 4;                 // softmax warpgroups; each takes 128 / kSoftWG keys of a step
constexpr int kSoftWarps = 4 * kSoftWG;
constexpr int kThreads = 32 * kSoftWarps + 64;  // + the producer warp and the MMA warp

template <int BS, int D>
struct Cfg {
  static constexpr int TM = 128;                 // query rows per tile
  static constexpr int R = TM / BS;              // block rows per tile
  static constexpr int NK = 128;                 // keys per step
  static constexpr int BPS = NK / BS;            // blocks per step
  static constexpr int KATOMS = D / 64;          // 128-byte column atoms of a D-wide row
  static constexpr int Q_BYTES = TM * D * 2;
  static constexpr int CH_BYTES = NK * D * 2;    // one K or V stage
  static constexpr int NKS = D == 64 ? 3 : 2;    // K stages
  static constexpr int NVS = D == 64 ? 3 : 2;    // V stages
  static constexpr int OFF_Q = 0;                // two Q buffers
  static constexpr int OFF_K = 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NKS * CH_BYTES;
  static constexpr int OFF_CTRL = OFF_V + NVS * CH_BYTES;
  static constexpr uint32_t TMEM_COLS = 512;
  // S buffers in TMEM: the MMA issuer runs NS - 1 steps ahead of the
  // softmax.  Three fit beside two O accumulators for d = 64; for d = 128 the
  // second O buffer (the next tile's PVs overlap this tile's epilogue) was
  // measured to matter more than a third S buffer.
  static constexpr int NS = D == 64 ? 3 : 2;
  static constexpr uint32_t TMEM_O = NS * 128;   // O accumulators follow the S buffers
  static constexpr int OB = 2;                   // tiles whose O fit side by side
  static_assert((Q_BYTES % 1024) == 0 && (CH_BYTES % 1024) == 0, "1024-byte aligned stages");
  static_assert(TMEM_O + OB * D <= TMEM_COLS, "TMEM layout");
  static_assert(TM == NK, "Q and K tiles share one slice-offset formula");
};

constexpr int kMaxGrid = 256;               // CTAs per launch (the host caps the grid)
constexpr int kMaxHeavyGroups = 2 * kMaxGrid;

// This CTA's work (see `schedule`).
struct Sched {
  long long heavy[2];               // this CTA's heavy tiles
  long long n_light;                // light tiles in all
  long long kh;                     // heavy tiles in all
  long long scan[kThreads / 32];
  int n_heavy;
  int skip;                         // rounds of light tiles a CTA holding a heavy tile sits out
  int kg;                           // heavy groups per batch element
  // producer-side cursor
  int next_heavy;
  long long round;                  // next round of light tiles
  long long hp;                     // heavy tiles known to lie before the current light tile
  int heavy_hg[kMaxHeavyGroups];    // heavy groups of one batch element, in order
  int heavy_cost[kMaxHeavyGroups];
};

struct Ctrl {
  uint64_t bm_full[2], bm_empty[2];
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint64_t s_full[3], p_full[3], pv_done[3];
  uint64_t o_full[2], o_empty[2];
  uint64_t xbar[2][4];  // [exchange parity][lane quadrant]: one warp of each softmax warpgroup
  uint64_t final_bar;
  long long tile[2];  // tile index of each bitmap buffer, -1 = no more work
  int n[2];           // union size (blocks) of each bitmap buffer
  Sched sched;
  uint32_t tmem_base;
  AbortFlag abort;
  float red[2][kSoftWG][128];  // [exchange parity][warpgroup][row]: partial row max or sum
  uint32_t bitmap[2][5 * kMaxBitmapWords];  // R block-row maps, then their union
};

// Estimated cost of tile group (h, g) in blocks: the longest of its rows, plus
// one step for the per-tile overhead.
template <int BS>
__device__ __forceinline__ long long group_cost(const FwdArgs& a, long long hg) {
  constexpr int R = 128 / BS;
  const long long h = hg / a.G;
  const int g = static_cast<int>(hg - h * a.G);
  const int32_t* rp = a.row_ptr + h * a.M;
  int mx = 0;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int r = g * R + i;
    if (r < a.M) mx = max(mx, __ldg(rp + r + 1) - __ldg(rp + r));
  }
  return mx + R;
}

// Block-wide exclusive scan of v (every thread calls it); *total = sum over the CTA.
__device__ __forceinline__ long long block_scan(long long v, long long* total, long long* buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  __syncthreads();  // buf is free again
  if (lane == 31) buf[warp] = incl;
  __syncthreads();
  long long base = 0, tot = 0;
  for (int w = 0; w < kThreads / 32; ++w) {
    const long long x = buf[w];
    if (w < warp) base += x;
    tot += x;
  }
  *total = tot;
  return base + incl - v;
}

// All threads: this CTA's share of the tiles (the tile schedule).
//
// Tile T = (b*H + h)*G + g; its cost is group_cost of group hg = h*G + g (the
// pattern is shared across b).  Every CTA computes the same plan:
//  1. total = sum of the tile costs; a tile is heavy when its cost exceeds
//     thr = total / (2*grid), half of one CTA's share, so there are fewer than
//     2*grid heavy tiles.  Heavy tile k (in tile order) goes to CTA k mod grid.
//  2. The other ("light") tiles, in tile order, are dealt out in rounds of
//     one tile per CTA, so that the CTAs work on neighbouring tiles at any
//     time and share the K/V blocks those tiles read in L2.
//  3. When there are at most `grid` heavy tiles, the CTAs holding one sit out
//     the first `skip` rounds, skip = average heavy cost / average light cost.
template <int BS>
__device__ void schedule(const FwdArgs& a, Ctrl* ctl) {
  Sched& sd = ctl->sched;
  const int tid = threadIdx.x;
  const long long HG = static_cast<long long>(a.H) * a.G;
  const long long seg = (HG + kThreads - 1) / kThreads;
  const long long lo = min(HG, tid * seg), hi = min(HG, lo + seg);
  const long long nb = a.num_tiles / HG;
  const long long grid = gridDim.x;
  const long long c = blockIdx.x;

  long long sum = 0;
  for (long long hg = lo; hg < hi; ++hg) sum += group_cost<BS>(a, hg);
  long long per_b;
  block_scan(sum, &per_b, sd.scan);
  const long long total = per_b * nb;
  const long long thr = total / (2 * grid);

  long long n_hv = 0, hsum = 0;
  for (long long hg = lo; hg < hi; ++hg) {
    const long long cst = group_cost<BS>(a, hg);
    if (cst > thr) {
      ++n_hv;
      hsum += cst;
    }
  }
  long long Kg, Hper;
  long long hexcl = block_scan(n_hv, &Kg, sd.scan);
  block_scan(hsum, &Hper, sd.scan);
  for (long long hg = lo; hg < hi && n_hv > 0; ++hg) {
    const long long cst = group_cost<BS>(a, hg);
    if (cst > thr) {
      sd.heavy_hg[hexcl] = static_cast<int>(hg);
      sd.heavy_cost[hexcl] = static_cast<int>(cst);
      ++hexcl;
    }
  }
  if (tid == 0) {
    const long long Kh = Kg * nb;  // < 2*grid <= kMaxHeavyGroups
    const long long n_light = a.num_tiles - Kh;
    int nh = 0;
    for (long long k = c; k < Kh && nh < 2; k += grid)
      sd.heavy[nh++] = (k / Kg) * HG + sd.heavy_hg[k % Kg];
    long long skip = 0;
    if (Kh > 0 && Kh <= grid && n_light > 0) {
      const double heavy_avg = static_cast<double>(Hper * nb) / Kh;
      const double light_avg = static_cast<double>(total - Hper * nb) / n_light;
      skip = static_cast<long long>(heavy_avg / light_avg + 0.5);
      const long long most = n_light / (grid - Kh > 0 ? grid - Kh : 1);
      if (skip > most) skip = most;
      if (grid - Kh <= 0) skip = 0;
    }
    sd.n_heavy = nh;
    sd.kh = Kh;
    sd.kg = static_cast<int>(Kg);
    sd.n_light = n_light;
    sd.skip = static_cast<int>(skip);
    sd.next_heavy = 0;
    sd.round = 0;
    sd.hp = 0;
  }
  __syncthreads();
}

// Next tile of this CTA (producer lane 0), -1 when none is left: its heavy
// tiles first, then its light tiles in increasing order.
template <int BS>
__device__ __forceinline__ long long next_tile(const FwdArgs& a, Sched& sd) {
  if (sd.next_heavy < sd.n_heavy) return sd.heavy[sd.next_heavy++];
  const long long grid = gridDim.x, c = blockIdx.x;
  const long long Kh = sd.kh;
  const bool skipping = sd.skip > 0;             // at most grid heavy tiles, CTAs 0..Kh-1 hold one
  const long long others = grid - Kh;            // CTAs without a heavy tile
  const long long k = sd.round++;
  long long i;                                   // index among the light tiles
  if (!skipping) {
    i = k * grid + c;
  } else if (k < sd.skip) {
    if (c < Kh) {                                // sits out the first rounds
      sd.round = sd.skip + 1;
      i = static_cast<long long>(sd.skip) * others + c;
    } else {
      i = k * others + (c - Kh);
    }
  } else {
    i = static_cast<long long>(sd.skip) * others + (k - sd.skip) * grid + c;
  }
  if (i >= sd.n_light) return -1;
  // Light tile i is tile i + (heavy tiles before it); the heavy tiles are in
  // increasing tile order and i only grows, so the count is kept across calls.
  const long long HG = static_cast<long long>(a.H) * a.G;
  long long t = i + sd.hp;
  while (sd.hp < Kh && (sd.hp / sd.kg) * HG + sd.heavy_hg[sd.hp % sd.kg] <= t) {
    ++sd.hp;
    t = i + sd.hp;
  }
  return t;
}

// ------------------------------------------------------------ producer warp
// Builds each tile's bitmaps (all lanes) and issues the TMA loads (lane 0) in
// the order the MMA issuer consumes them: Q, then K(j), V(j) for every step.
template <int BS, int D>
__device__ void load_role(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                          const FwdArgs& a, uint8_t* smem, Ctrl* ctl) {
  using C = Cfg<BS, D>;
  const int lane = threadIdx.x & 31;
  uint32_t q_loads = 0, k_loads = 0, v_loads = 0;
  bool ok = true;
  if (lane == 0) {
    prefetch_tensormap(tmQ);
    prefetch_tensormap(tmK);
    prefetch_tensormap(tmV);
  }
  for (int t = 0;; ++t) {
    const int buf = t & 1;
    int w_ok = 1;
    long long tile = -1;
    if (lane == 0) {
      w_ok = wait_bounded(&ctl->bm_empty[buf], ((t >> 1) & 1) ^ 1, &ctl->abort);
      if (w_ok) tile = next_tile<BS>(a, ctl->sched);
    }
    if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
    tile = __shfl_sync(0xffffffffu, tile, 0);

    uint32_t* bm = ctl->bitmap[buf];
    const int W = a.W;
    long long bh = 0;
    int n = 0;
    if (tile >= 0) {
      for (int w = lane; w < (C::R + 1) * W; w += 32) bm[w] = 0u;
      __syncwarp();
      bh = tile / a.G;
      const int g = static_cast<int>(tile - bh * a.G);
      const int h = static_cast<int>(bh % a.H);
      for (int i = 0; i < C::R; ++i) {
        const int r = g * C::R + i;
        if (r >= a.M) break;
        const int beg = __ldg(a.row_ptr + (static_cast<long long>(h) * a.M + r));
        const int end = __ldg(a.row_ptr + (static_cast<long long>(h) * a.M + r + 1));
        if (end < beg) {
          if (lane == 0) atomicOr(&g_status, BSA_STATUS_BAD_ROW_PTR);
          continue;
        }
        for (int p = beg + lane; p < end; p += 32) {
          const int j = __ldg(a.col_idx + p);
          if (j < 0 || j >= a.M) {
            atomicOr(&g_status, BSA_STATUS_BAD_COLUMN);
            continue;
          }
          if (a.causal && j > r) continue;  // every key of the block is after every query
          atomicOr(&bm[i * W + (j >> 5)], 1u << (j & 31));
          atomicOr(&bm[C::R * W + (j >> 5)], 1u << (j & 31));
        }
      }
      __threadfence_block();
      __syncwarp();
      n = union_count(bm + C::R * W, W);
    }
    if (lane == 0) {
      ctl->tile[buf] = tile;
      ctl->n[buf] = n;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->bm_full[buf]);
    if (tile < 0) break;
    if (n == 0) continue;

    if (lane == 0) {
      const int g = static_cast<int>(tile - bh * a.G);
      const uint32_t qb = q_loads & 1;
      ok = wait_bounded(&ctl->q_empty[qb], ((q_loads >> 1) & 1) ^ 1, &ctl->abort);
      if (ok) {
        mbar_arrive_expect_tx(&ctl->q_full[qb], C::Q_BYTES);
#pragma unroll
        for (int ka = 0; ka < C::KATOMS; ++ka)
          tma_load_3d(smem + C::OFF_Q + qb * C::Q_BYTES + ka * (C::TM * 128), tmQ, &ctl->q_full[qb],
                      ka * 64, g * C::TM, static_cast<int>(bh));
        ++q_loads;
      }
      BitIter it(bm + C::R * W, W);
      const int steps = (n + C::BPS - 1) / C::BPS;
      for (int j = 0; ok && j < steps; ++j) {
        int row0[C::BPS];  // first token of each block of the step; N (all out of range) pads
#pragma unroll
        for (int b = 0; b < C::BPS; ++b) {
          const int jb = it.next();
          row0[b] = jb >= 0 ? jb * BS : a.N;
        }
        const uint32_t ks = k_loads % C::NKS;
        ok = wait_bounded(&ctl->k_empty[ks], ((k_loads / C::NKS) & 1) ^ 1, &ctl->abort);
        if (!ok) break;
        mbar_arrive_expect_tx(&ctl->k_full[ks], C::CH_BYTES);
#pragma unroll
        for (int b = 0; b < C::BPS; ++b)
#pragma unroll
          for (int ka = 0; ka < C::KATOMS; ++ka)
            tma_load_3d(smem + C::OFF_K + ks * C::CH_BYTES + ka * (C::NK * 128) + b * (BS * 128), tmK,
                        &ctl->k_full[ks], ka * 64, row0[b], static_cast<int>(bh));
        ++k_loads;
        const uint32_t vs = v_loads % C::NVS;
        ok = wait_bounded(&ctl->v_empty[vs], ((v_loads / C::NVS) & 1) ^ 1, &ctl->abort);
        if (!ok) break;
        mbar_arrive_expect_tx(&ctl->v_full[vs], C::CH_BYTES);
#pragma unroll
        for (int b = 0; b < C::BPS; ++b)
#pragma unroll
          for (int ka = 0; ka < C::KATOMS; ++ka)
            tma_load_3d(smem + C::OFF_V + vs * C::CH_BYTES + ka * (C::NK * 128) + b * (BS * 128), tmV,
                        &ctl->v_full[vs], ka * 64, row0[b], static_cast<int>(bh));
        ++v_loads;
      }
    }
    if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { ok = false; break; }
  }
  // On an early exit, let every copy already issued land before the CTA ends.
  if (!ok && lane == 0) {
    for (uint32_t b = 0; b < 2; ++b)
      if (q_loads > b) {
        const uint32_t last = b + 2 * ((q_loads - 1 - b) / 2);
        wait_drain(&ctl->q_full[b], (last >> 1) & 1);
      }
    for (uint32_t st = 0; st < C::NKS; ++st)
      if (k_loads > st) {
        const uint32_t last = st + C::NKS * ((k_loads - 1 - st) / C::NKS);
        wait_drain(&ctl->k_full[st], (last / C::NKS) & 1);
      }
    for (uint32_t st = 0; st < C::NVS; ++st)
      if (v_loads > st) {
        const uint32_t last = st + C::NVS * ((v_loads - 1 - st) / C::NVS);
        wait_drain(&ctl->v_full[st], (last / C::NVS) & 1);
      }
  }
  __syncwarp();
}

// ---------------------------------------------------------------- MMA issuer
// Issue order within a tile of n steps: S(0), S(1), then for j = 0..n-1:
// O += P(j) V(j) and S(j+2).  MMAs of one thread run in issue order, so S(j+2)
// overwrites S(j)/P(j) only after the PV of step j has read P(j), and each
// commit also reports every MMA issued before it.
template <int BS, int D>
__device__ void mma_role(const FwdArgs& a, uint8_t* smem, Ctrl* ctl, uint32_t tmem) {
  using C = Cfg<BS, D>;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, C::NK, false, false);  // Q, K K-major
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);       // V MN-major
  const uint32_t q_base = smem_u32(smem + C::OFF_Q);
  const uint32_t k_base = smem_u32(smem + C::OFF_K);
  const uint32_t v_base = smem_u32(smem + C::OFF_V);
  uint32_t k_cons = 0, v_cons = 0, q_uses = 0, o_tiles = 0, gstep = 0;
  bool ok = true;
  for (int t = 0; ok; ++t) {
    const int buf = t & 1;
    if (!wait_bounded(&ctl->bm_full[buf], (t >> 1) & 1, &ctl->abort)) break;
    const long long tile = ctl->tile[buf];
    const int n = ctl->n[buf];
    mbar_arrive(&ctl->bm_empty[buf]);
    if (tile < 0) break;
    if (n == 0) continue;
    const int steps = (n + C::BPS - 1) / C::BPS;
    const uint32_t qb = q_uses & 1;
    if (!wait_bounded(&ctl->q_full[qb], (q_uses >> 1) & 1, &ctl->abort)) break;
    ++q_uses;
    const uint32_t ob = o_tiles % C::OB;
    const uint32_t t_o = tmem + C::TMEM_O + ob * D;
    const uint32_t q_tile = q_base + qb * C::Q_BYTES;

    auto issue_qk = [&](int j) -> bool {
      const uint32_t sb = (gstep + j) % C::NS;
      const uint32_t ks = k_cons % C::NKS;
      if (!wait_bounded(&ctl->k_full[ks], (k_cons / C::NKS) & 1, &ctl->abort)) return false;
      tc_fence_after();
      // Descriptors of consecutive K=16 slices differ only in the start
      // address field (address >> 4), so they are a base plus a constant.
      const uint64_t ad0 = sdesc_sw128(q_tile, 16, 1024);
      const uint64_t bd0 = sdesc_sw128(k_base + ks * C::CH_BYTES, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk >> 2) * (C::TM * 128) + (kk & 3) * 32) >> 4;  // TM == NK
        umma_bf16_ss(tmem + sb * 128, ad0 + off, bd0 + off, kIdescQK, kk > 0 ? 1u : 0u);
      }
      umma_commit(&ctl->k_empty[ks]);
      umma_commit(&ctl->s_full[sb]);
      if (j == steps - 1) umma_commit(&ctl->q_empty[qb]);
      ++k_cons;
      return true;
    };
    auto issue_pv = [&](int j) -> bool {
      const uint32_t gs = gstep + j, sb = gs % C::NS;
      if (!wait_bounded(&ctl->p_full[sb], (gs / C::NS) & 1, &ctl->abort)) return false;
      const uint32_t vs = v_cons % C::NVS;
      if (!wait_bounded(&ctl->v_full[vs], (v_cons / C::NVS) & 1, &ctl->abort)) return false;
      if (j == 0 && o_tiles >= C::OB &&
          !wait_bounded(&ctl->o_empty[ob], ((o_tiles - C::OB) / C::OB) & 1, &ctl->abort))
        return false;
      tc_fence_after();
      const uint64_t bd0 = sdesc_sw128(v_base + vs * C::CH_BYTES, C::NK * 128, 1024);
      const uint32_t a0 = tmem + sb * 128;
#pragma unroll
      for (int kk = 0; kk < C::NK / 16; ++kk) {
        // P of keys 16kk..16kk+15: warpgroup kk/2 packs its 32 keys into the
        // first 16 of its 32 score columns.
        const uint32_t a_col = (kk >> 1) * 32 + (kk & 1) * 8;
        umma_bf16_ts(t_o, a0 + a_col, bd0 + ((kk * 16 * 128) >> 4), kIdescPV,
                     (j > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&ctl->v_empty[vs]);
      umma_commit(&ctl->pv_done[sb]);
      if (j == steps - 1) umma_commit(&ctl->o_full[ob]);
      ++v_cons;
      return true;
    };

    ok = issue_qk(0);
    for (int j = 1; ok && j < C::NS && j < steps; ++j) ok = issue_qk(j);
    for (int j = 0; ok && j < steps; ++j)
      ok = issue_pv(j) && (j + C::NS >= steps || issue_qk(j + C::NS));
    gstep += steps;
    ++o_tiles;
  }
  // Every MMA issued must complete before the TMEM is released.
  umma_commit(&ctl->final_bar);
  wait_drain(&ctl->final_bar, 0);
}

// ------------------------------------------------------------ softmax warps
// Warpgroup `qt` handles keys 32 qt .. 32 qt + 31 of every step (one group of
// 32 TMEM columns) for all 128 rows, and O columns [qt d/4, (qt+1) d/4) in
// the epilogue.  The kSoftWG warps that hold the same rows (one per
// warpgroup, TMEM lane quadrant wq) exchange their partial row maxima each
// step and their partial sums at the end of a tile.
template <int BS, int D>
__device__ void softmax_role(int qt, const FwdArgs& a, Ctrl* ctl, uint32_t tmem) {
  using C = Cfg<BS, D>;
  constexpr int QD = D / kSoftWG;              // O columns of this warpgroup (16 or 32)
  const int wq = (threadIdx.x >> 5) & 3;       // TMEM lane quadrant
  const int lane = threadIdx.x & 31;
  const int row = wq * 32 + lane;              // query row of the tile
  const int sub = row / BS;                    // block row of the tile this thread belongs to
  const int qq = row % BS;                     // position inside that block row
  const uint32_t t_lane = static_cast<uint32_t>(wq * 32) << 16;
  const float sl2 = a.scale_log2;
  constexpr float kNegInf = -INFINITY;
  const int b_mine = (qt * 32) / BS;           // block of the step holding this group
  const int c0 = (qt * 32) % BS;               // first column of the group inside its block
  uint32_t gstep = 0, o_tiles = 0, n_ex = 0;
  // The warps sharing these rows have written their values for exchange
  // n_ex: each arrives on xbar[n_ex & 1][wq] (kSoftWG arrivals complete it)
  // and waits for the phase (bounded).  Values live in buffer n_ex & 1, so
  // the next write to a buffer comes after every partner has passed the
  // exchange that read it.
  auto exchange = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->xbar[n_ex & 1][wq]);
    return warp_wait(&ctl->xbar[n_ex & 1][wq], (n_ex >> 1) & 1, &ctl->abort);
  };

  for (int t = 0;; ++t) {
    const int buf = t & 1;
    if (!warp_wait(&ctl->bm_full[buf], (t >> 1) & 1, &ctl->abort)) return;
    const long long tile = ctl->tile[buf];
    const int n = ctl->n[buf];
    if (tile < 0) return;
    const uint32_t* bm = ctl->bitmap[buf];
    const uint32_t* mine = bm + sub * a.W;
    const long long bh = tile / a.G;
    const int g = static_cast<int>(tile - bh * a.G);
    const int r_sub = g * C::R + sub;
    const bool row_ok = r_sub < a.M;
    const int steps = (n + C::BPS - 1) / C::BPS;
    const long long qtok = static_cast<long long>(g) * C::TM + row;
    uint4* orow = reinterpret_cast<uint4*>(a.O + (bh * a.N + qtok) * D + qt * QD);

    if (n == 0) {
      if (row_ok) {
#pragma unroll
        for (int c = 0; c < QD / 8; ++c) orow[c] = make_uint4(0u, 0u, 0u, 0u);
        if (qt == 0) a.LSE[bh * a.N + qtok] = kNegInf;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->bm_empty[buf]);
      continue;
    }

    float m_used = kNegInf;  // running max, log2 units of the scaled score (same in every warpgroup)
    float l = 0.f;           // this warpgroup's running sum of 2^(s - m_used)
    const uint32_t ob = o_tiles % C::OB;
    BitIter it(bm + C::R * a.W, a.W);
    for (int j = 0; j < steps; ++j) {
      const uint32_t gs = gstep + j, sb = gs % C::NS;
      bool valid = false, diag = false;  // this row holds the group's block / it is the diagonal
#pragma unroll
      for (int b = 0; b < C::BPS; ++b) {
        const int jb = it.next();
        if (b != b_mine) continue;
        valid = row_ok && jb >= 0 && ((mine[jb >> 5] >> (jb & 31)) & 1u);
        diag = a.causal && jb == r_sub;
      }
      if (!warp_wait(&ctl->s_full[sb], (gs / C::NS) & 1, &ctl->abort)) return;
      tc_fence_after();
      const uint32_t t_s = tmem + t_lane + sb * 128 + qt * 32;
      uint32_t u[32];
      float pmax = kNegInf;
      if (valid) {  // uniform over the warp
        tmem_ld32(t_s, u);
        tmem_wait_ld();
        reg_fence32(u);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float v = __uint_as_float(u[c]) * sl2;
          if (diag && c0 + c > qq) v = kNegInf;  // key after the query (diagonal block only)
          u[c] = __float_as_uint(v);
          pmax = fmaxf(pmax, v);
        }
      }
      // Row maximum over all warpgroups.
      ctl->red[n_ex & 1][qt][row] = pmax;
      if (!exchange()) return;
      float mx = kNegInf;
#pragma unroll
      for (int o = 0; o < kSoftWG; ++o) mx = fmaxf(mx, ctl->red[n_ex & 1][o][row]);
      ++n_ex;

      // Lazy rescale: the running maximum moves only when the step's maximum
      // exceeds it by more than the threshold (P stays <= 2^8 otherwise).
      float factor = 1.f;
      bool need_rescale = false;
      if (mx > m_used + kRescaleThreshold) {
        if (m_used != kNegInf) {
          need_rescale = true;
          factor = ex2_approx(m_used - mx);
        }
        m_used = mx;
      }
      if (__any_sync(0xffffffffu, need_rescale)) {
        // O must hold every PV up to the previous step.
        const uint32_t pg = gs - 1;
        if (!warp_wait(&ctl->pv_done[pg % C::NS], (pg / C::NS) & 1, &ctl->abort)) return;
        tc_fence_after();
        const uint32_t t_o = tmem + t_lane + C::TMEM_O + ob * D + qt * QD;
        uint32_t w[32];
        if constexpr (QD == 32) tmem_ld32(t_o, w);
        else tmem_ld16(t_o, *reinterpret_cast<uint32_t(*)[16]>(&w[0]));
        tmem_wait_ld();
        reg_fence32(w);
#pragma unroll
        for (int i = 0; i < QD; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * factor);
        if constexpr (QD == 32) tmem_st32(t_o, w);
        else tmem_st16(t_o, *reinterpret_cast<uint32_t(*)[16]>(&w[0]));
      }
      l *= factor;

      uint32_t pk[16];
      if (valid) {
        const float mu = m_used == kNegInf ? 0.f : m_used;
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = ex2_approx(__uint_as_float(u[c]) - mu);
          const float p1 = ex2_approx(__uint_as_float(u[c + 1]) - mu);
          rs += p0;
          rs += p1;
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        l += rs;
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = 0u;
      }
      tmem_st16(t_s, pk);  // P of this group's 32 keys, over its first 16 columns
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[sb]);
    }

    // Epilogue: O / l in bf16 (this warpgroup's columns) and LSE = (m + log2 l) ln 2.
    ctl->red[n_ex & 1][qt][row] = l;
    if (!exchange()) return;
    float lt = 0.f;
#pragma unroll
    for (int o = 0; o < kSoftWG; ++o) lt += ctl->red[n_ex & 1][o][row];
    ++n_ex;
    if (!warp_wait(&ctl->o_full[ob], (o_tiles / C::OB) & 1, &ctl->abort)) return;
    tc_fence_after();
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
    const uint32_t t_o = tmem + t_lane + C::TMEM_O + ob * D + qt * QD;
    uint32_t w[32];
    if constexpr (QD == 32) tmem_ld32(t_o, w);
    else tmem_ld16(t_o, *reinterpret_cast<uint32_t(*)[16]>(&w[0]));
    tmem_wait_ld();
    reg_fence32(w);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&ctl->o_empty[ob]);
      mbar_arrive(&ctl->bm_empty[buf]);
    }
    if (row_ok) {
#pragma unroll
      for (int q = 0; q < QD / 8; ++q) {
        uint4 v;
        v.x = pack_bf16x2(__uint_as_float(w[q * 8 + 0]) * inv, __uint_as_float(w[q * 8 + 1]) * inv);
        v.y = pack_bf16x2(__uint_as_float(w[q * 8 + 2]) * inv, __uint_as_float(w[q * 8 + 3]) * inv);
        v.z = pack_bf16x2(__uint_as_float(w[q * 8 + 4]) * inv, __uint_as_float(w[q * 8 + 5]) * inv);
        v.w = pack_bf16x2(__uint_as_float(w[q * 8 + 6]) * inv, __uint_as_float(w[q * 8 + 7]) * inv);
        orow[q] = v;
      }
      if (qt == 0)
        a.LSE[bh * a.N + qtok] = lt > 0.f ? (m_used + __log2f(lt)) * 0.69314718055994531f : kNegInf;
    }
    gstep += steps;
    ++o_tiles;
  }
}

template <int BS, int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdArgs args) {
  using C = Cfg<BS, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Ctrl* ctl = reinterpret_cast<Ctrl*>(smem + C::OFF_CTRL);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->bm_full[b], 1);
      mbar_init(&ctl->bm_empty[b], kSoftWarps + 1);  // the softmax warps + the MMA issuer
      mbar_init(&ctl->q_full[b], 1);
      mbar_init(&ctl->q_empty[b], 1);

      mbar_init(&ctl->o_full[b], 1);
      mbar_init(&ctl->o_empty[b], kSoftWarps);
      for (int q = 0; q < 4; ++q) mbar_init(&ctl->xbar[b][q], kSoftWG);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(&ctl->s_full[s], 1);
      mbar_init(&ctl->p_full[s], kSoftWarps);
      mbar_init(&ctl->pv_done[s], 1);
      mbar_init(&ctl->k_full[s], 1);
      mbar_init(&ctl->k_empty[s], 1);
      mbar_init(&ctl->v_full[s], 1);
      mbar_init(&ctl->v_empty[s], 1);
    }
    mbar_init(&ctl->final_bar, 1);
    ctl->abort.v = 0;
    fence_mbar_init();
  }
  if (warp == kSoftWarps + 1) {
    tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  schedule<BS>(args, ctl);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp < kSoftWarps) {
    softmax_role<BS, D>(warp >> 2, args, ctl, tmem);
    __syncwarp();
  } else if (warp == kSoftWarps) {
    load_role<BS, D>(&tmQ, &tmK, &tmV, args, smem, ctl);
  } else if (warp == kSoftWarps + 1) {
    if ((threadIdx.x & 31) == 0) mma_role<BS, D>(args, smem, ctl, tmem);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kSoftWarps + 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace rows
}  // namespace bsa
