// bsa_fwd_pp.cuh -- two-slot ("ping-pong") forward kernel, every block size.
//
// A tile is 128 query rows = R = 128 / block_size consecutive block rows of
// one (b, h).  It walks the union of its rows' column lists in steps of 128
// keys (128 / block_size blocks gathered into one shared-memory stage):
//
//   S = Q K_step^T            tcgen05.mma, M=128 queries, N=128 keys, K=d
//   P = 2^(S*scale*log2e - m) fp32 in registers, written back to TMEM as bf16
//   O += P V_step             tcgen05.mma with A = P read from TMEM, N=d
//
// A block row that does not hold a block of the step gets P = 0 there and its
// statistics skip it, so every row sums exactly over its own blocks ("Block
// Sparse Attention with Log-Linear Complexity", section 3.3).  Membership is
// uniform over a warp for every block size, so the scores of such blocks are
// neither loaded from TMEM nor exponentiated.
//
// One persistent CTA per SM holds two independent tile slots.  Each slot has
// its own S and O in TMEM and its own softmax warpgroup, in which thread i
// owns query row i of the tile (TMEM lane i): the row maximum and sum need
// no exchange between threads.  The MMA warp alternates between the slots,
// so the tensor core computes one slot's P V and next scores while the other
// slot's warpgroup turns its scores into probabilities.  Roles (384 threads):
//   warps 0-3   softmax and epilogue of slot 0
//   warps 4-7   softmax and epilogue of slot 1
//   warp 8      TMA loads of Q, K, V for both slots, in the MMA's order
//   warp 9      tcgen05.mma issuer (and owner of the 512 TMEM columns)
//   warps 10-11 tile builders of slot 0 / slot 1: take the slot's next tile
//               from the schedule and turn its CSR rows into block bitmaps
//
// TMEM columns: S of slot s in [128 s, +128), P (bf16 pairs) over its first
// 64 columns once the scores are in registers; O of slot s in [256 + d s, +d).
//
// Work split (`schedule`): the 2 * grid slots are scheduled as independent
// workers.  Tiles whose estimated cost exceeds half of one slot's share are
// dealt out first, one per slot; the other tiles go out in round-robin
// rounds, so that concurrently running slots work on neighbouring tiles and
// share their K/V blocks in L2.
#pragma once

#include "bsa_common.cuh"

namespace bsa {
namespace pp {

constexpr int kSlots = 2;
constexpr int kWarps = 12;
constexpr int kThreads = 32 * kWarps;
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kBuildWarp = 10;              // builder of slot s is warp kBuildWarp + s
constexpr int kLaunchRegs = 168;            // 65536 / kThreads, rounded down to a multiple of 8
constexpr int kSoftRegs = 208;
constexpr int kOtherRegs = 88;
static_assert(4 * 32 * (kSlots * kSoftRegs + kOtherRegs) <= kThreads * kLaunchRegs,
              "register split exceeds the launch's registers");
static_assert(kThreads * kLaunchRegs <= 65536, "registers per SM");

constexpr int kMaxGrid = 160;               // CTAs per launch (the host caps the grid)
constexpr int kMaxVirt = kSlots * kMaxGrid; // slots scheduled as workers
constexpr int kMaxHeavyGroups = 2 * kMaxVirt;

template <int BS, int D>
struct Cfg {
  static constexpr int TM = 128;                 // query rows per tile
  static constexpr int R = TM / BS;              // block rows per tile
  static constexpr int NK = 128;                 // keys per step
  static constexpr int BPS = NK / BS;            // blocks per step
  static constexpr int KATOMS = D / 64;          // 128-byte column atoms of a D-wide row
  static constexpr int Q_BYTES = TM * D * 2;
  static constexpr int CH_BYTES = NK * D * 2;    // one K or V stage
  static constexpr int QB = D == 64 ? 2 : 1;     // Q buffers per slot
  static constexpr int NKS = D == 64 ? 4 : 2;    // K stages (shared by both slots)
  static constexpr int NVS = D == 64 ? 4 : 2;    // V stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = kSlots * QB * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NKS * CH_BYTES;
  static constexpr int OFF_CTRL = OFF_V + NVS * CH_BYTES;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TMEM_O = 2 * 128;    // O of slot s at TMEM_O + D s
  static_assert((Q_BYTES % 1024) == 0 && (CH_BYTES % 1024) == 0, "1024-byte aligned stages");
  static_assert(TMEM_O + kSlots * D <= TMEM_COLS, "TMEM layout");
  static_assert(TM == NK, "Q and K tiles share one slice-offset formula");
};

// The plan every CTA computes identically (see `schedule`).
struct Plan {
  long long n_light;                // light tiles in all
  long long kh;                     // heavy tiles in all
  long long scan[kWarps];
  int skip;                         // rounds of light tiles a slot holding a heavy tile sits out
  int kg;                           // heavy groups per batch element
  int heavy_hg[kMaxHeavyGroups];    // heavy groups of one batch element, in order
};

// One slot's position in the plan (its builder warp advances it).
struct Cursor {
  long long heavy[2];               // this slot's heavy tiles
  long long round;                  // next round of light tiles
  long long hp;                     // heavy tiles known to lie before the current light tile
  int n_heavy;
  int next_heavy;
};

struct TileInfo {
  long long tile;  // tile index, -1 = no more work for this slot
  int n;           // union size in blocks
  int pad;
};

struct Ctrl {
  uint64_t t_full[kSlots][2], t_empty[kSlots][2];
  uint64_t q_full[kSlots][2], q_empty[kSlots][2];
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[kSlots], p_full[kSlots], o_full[kSlots];
  uint64_t final_bar;
  TileInfo info[kSlots][2];
  Cursor cur[kSlots];
  uint32_t tmem_base;
  AbortFlag abort;
  Plan plan;
};

// 32-bit words of one tile's bitmaps: R block-row maps, then their union.
template <int BS>
__host__ __device__ constexpr int bitmap_words(int W) {
  return (128 / BS + 1) * W;
}

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
  for (int w = 0; w < kWarps; ++w) {
    const long long x = buf[w];
    if (w < warp) base += x;
    tot += x;
  }
  *total = tot;
  return base + incl - v;
}

// All threads: the tile schedule, with the CTA's two slots as workers
// v = 2 * blockIdx.x + s among V = 2 * gridDim.x.
//
// Tile T = (b*H + h)*G + g; its cost is group_cost of group hg = h*G + g (the
// pattern is shared across b).  Every CTA computes the same plan:
//  1. total = sum of the tile costs; a tile is heavy when its cost exceeds
//     thr = total / (2V), half of one slot's share, so there are fewer than
//     2V heavy tiles.  Heavy tile k (in tile order) goes to slot k mod V.
//  2. The other ("light") tiles, in tile order, are dealt out in rounds of
//     one tile per slot.
//  3. When there are at most V heavy tiles, the slots holding one sit out
//     the first `skip` rounds, skip = average heavy cost / average light cost.
template <int BS>
__device__ void schedule(const FwdArgs& a, Ctrl* ctl) {
  Plan& pl = ctl->plan;
  const int tid = threadIdx.x;
  const long long HG = static_cast<long long>(a.H) * a.G;
  const long long seg = (HG + kThreads - 1) / kThreads;
  const long long lo = min(HG, tid * seg), hi = min(HG, lo + seg);
  const long long nb = a.num_tiles / HG;
  const long long V = static_cast<long long>(kSlots) * gridDim.x;

  long long sum = 0;
  for (long long hg = lo; hg < hi; ++hg) sum += group_cost<BS>(a, hg);
  long long per_b;
  block_scan(sum, &per_b, pl.scan);
  const long long total = per_b * nb;
  const long long thr = total / (2 * V);

  long long n_hv = 0, hsum = 0;
  for (long long hg = lo; hg < hi; ++hg) {
    const long long cst = group_cost<BS>(a, hg);
    if (cst > thr) {
      ++n_hv;
      hsum += cst;
    }
  }
  long long Kg, Hper;
  long long hexcl = block_scan(n_hv, &Kg, pl.scan);
  block_scan(hsum, &Hper, pl.scan);
  for (long long hg = lo; hg < hi && n_hv > 0; ++hg) {
    if (group_cost<BS>(a, hg) > thr) pl.heavy_hg[hexcl++] = static_cast<int>(hg);
  }
  if (tid == 0) {
    const long long Kh = Kg * nb;  // < 2V <= kMaxHeavyGroups
    const long long n_light = a.num_tiles - Kh;
    long long skip = 0;
    if (Kh > 0 && Kh <= V && n_light > 0 && V - Kh > 0) {
      const double heavy_avg = static_cast<double>(Hper * nb) / Kh;
      const double light_avg = static_cast<double>(total - Hper * nb) / n_light;
      skip = static_cast<long long>(heavy_avg / light_avg + 0.5);
      const long long most = n_light / (V - Kh);
      if (skip > most) skip = most;
    }
    pl.kh = Kh;
    pl.kg = static_cast<int>(Kg);
    pl.n_light = n_light;
    pl.skip = static_cast<int>(skip);
    for (int s = 0; s < kSlots; ++s) {
      Cursor& cu = ctl->cur[s];
      const long long v = static_cast<long long>(kSlots) * blockIdx.x + s;
      int nh = 0;
      for (long long k = v; k < Kh && nh < 2; k += V)
        cu.heavy[nh++] = (k / Kg) * HG + pl.heavy_hg[k % Kg];
      cu.n_heavy = nh;
      cu.next_heavy = 0;
      cu.round = 0;
      cu.hp = 0;
    }
  }
  __syncthreads();
}

// Next tile of slot worker v (one builder lane), -1 when none is left: its
// heavy tiles first, then its light tiles in increasing order.
__device__ __forceinline__ long long next_tile(const FwdArgs& a, const Plan& pl, Cursor& cu,
                                               long long v) {
  if (cu.next_heavy < cu.n_heavy) return cu.heavy[cu.next_heavy++];
  const long long V = static_cast<long long>(kSlots) * gridDim.x;
  const long long Kh = pl.kh;
  const bool skipping = pl.skip > 0;             // at most V heavy tiles, slots 0..Kh-1 hold one
  const long long others = V - Kh;               // slots without a heavy tile
  const long long k = cu.round++;
  long long i;                                   // index among the light tiles
  if (!skipping) {
    i = k * V + v;
  } else if (k < pl.skip) {
    if (v < Kh) {                                // sits out the first rounds
      cu.round = pl.skip + 1;
      i = static_cast<long long>(pl.skip) * others + v;
    } else {
      i = k * others + (v - Kh);
    }
  } else {
    i = static_cast<long long>(pl.skip) * others + (k - pl.skip) * V + v;
  }
  if (i >= pl.n_light) return -1;
  // Light tile i is tile i + (heavy tiles before it); the heavy tiles are in
  // increasing tile order and i only grows, so the count is kept across calls.
  const long long HG = static_cast<long long>(a.H) * a.G;
  long long t = i + cu.hp;
  while (cu.hp < Kh && (cu.hp / pl.kg) * HG + pl.heavy_hg[cu.hp % pl.kg] <= t) {
    ++cu.hp;
    t = i + cu.hp;
  }
  return t;
}

// ------------------------------------------------------------- tile builder
// Warp kBuildWarp + s: for each tile of slot s, the R block-row bitmaps and
// their union from the CSR rows, published in the slot's two-entry ring.
template <int BS, int D>
__device__ void build_role(int s, const FwdArgs& a, Ctrl* ctl, uint32_t* bitmaps) {
  using C = Cfg<BS, D>;
  const int lane = threadIdx.x & 31;
  const int W = a.W;
  const int BMW = bitmap_words<BS>(W);
  const long long v = static_cast<long long>(kSlots) * blockIdx.x + s;
  for (int t = 0;; ++t) {
    const int buf = t & 1;
    int w_ok = 1;
    long long tile = -1;
    if (lane == 0) {
      w_ok = wait_bounded(&ctl->t_empty[s][buf], ((t >> 1) & 1) ^ 1, &ctl->abort);
      if (w_ok) tile = next_tile(a, ctl->plan, ctl->cur[s], v);
    }
    if (!__shfl_sync(0xffffffffu, w_ok, 0)) return;
    tile = __shfl_sync(0xffffffffu, tile, 0);
    uint32_t* bm = bitmaps + (s * 2 + buf) * BMW;
    int n = 0;
    if (tile >= 0) {
      for (int w = lane; w < BMW; w += 32) bm[w] = 0u;
      __syncwarp();
      const long long bh = tile / a.G;
      const int g = static_cast<int>(tile - bh * a.G);
      const int h = static_cast<int>(bh % a.H);
      for (int i = 0; i < C::R; ++i) {
        const int r = g * C::R + i;
        if (r >= a.M) break;
        const int beg = __ldg(a.row_ptr + (static_cast<long long>(h) * a.M + r));
        const int end = __ldg(a.row_ptr + (static_cast<long long>(h) * a.M + r + 1));
        if (beg < 0 || end < beg) {
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
      ctl->info[s][buf].tile = tile;
      ctl->info[s][buf].n = n;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->t_full[s][buf]);
    if (tile < 0) return;
  }
}

// ------------------------------------------------------------ producer warp
// Lane 0 issues every TMA load in the order the MMA issuer consumes them:
// K(0) of each slot, then per slot in turn V(j) and the slot's next K (the
// next step of its tile, or step 0 of its next tile after that tile's Q).
template <int BS, int D>
__device__ void load_role(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                          const FwdArgs& a, uint8_t* smem, Ctrl* ctl, const uint32_t* bitmaps) {
  using C = Cfg<BS, D>;
  if ((threadIdx.x & 31) != 0) return;
  prefetch_tensormap(tmQ);
  prefetch_tensormap(tmK);
  prefetch_tensormap(tmV);
  const int W = a.W;
  const int BMW = bitmap_words<BS>(W);
  uint32_t q_loads[kSlots] = {0, 0}, k_loads = 0, v_loads = 0;
  int t[kSlots] = {0, 0}, steps[kSlots] = {0, 0}, j[kSlots] = {0, 0};
  bool active[kSlots] = {true, true};
  long long bh[kSlots] = {0, 0};
  int row0[kSlots][C::BPS];
  // union bitmap walk of each slot's current tile
  const uint32_t* ubits[kSlots] = {nullptr, nullptr};
  int uw[kSlots] = {0, 0};
  uint32_t ucur[kSlots] = {0, 0};
  bool ok = true;

  auto next_block = [&](int s) -> int {
    while (ucur[s] == 0) {
      if (++uw[s] >= W) return -1;
      ucur[s] = ubits[s][uw[s]];
    }
    const int b = __ffs(ucur[s]) - 1;
    ucur[s] &= ucur[s] - 1;
    return uw[s] * 32 + b;
  };
  // Moves slot s to its next non-empty tile and loads that tile's Q.
  auto next_tile_of = [&](int s) -> bool {
    for (;;) {
      const int buf = t[s] & 1;
      if (!wait_bounded(&ctl->t_full[s][buf], (t[s] >> 1) & 1, &ctl->abort)) return false;
      const long long tile = ctl->info[s][buf].tile;
      const int n = ctl->info[s][buf].n;
      if (tile < 0) {
        active[s] = false;
        return true;
      }
      if (n == 0) {
        mbar_arrive(&ctl->t_empty[s][buf]);
        ++t[s];
        continue;
      }
      bh[s] = tile / a.G;
      const int g = static_cast<int>(tile - bh[s] * a.G);
      ubits[s] = bitmaps + (s * 2 + buf) * BMW + C::R * W;
      uw[s] = 0;
      ucur[s] = ubits[s][0];
      steps[s] = (n + C::BPS - 1) / C::BPS;
      j[s] = 0;
      const uint32_t qb = q_loads[s] % C::QB;
      if (!wait_bounded(&ctl->q_empty[s][qb], ((q_loads[s] / C::QB) & 1) ^ 1, &ctl->abort))
        return false;
      mbar_arrive_expect_tx(&ctl->q_full[s][qb], C::Q_BYTES);
      uint8_t* qdst = smem + C::OFF_Q + (s * C::QB + qb) * C::Q_BYTES;
#pragma unroll
      for (int ka = 0; ka < C::KATOMS; ++ka)
        tma_load_3d(qdst + ka * (C::TM * 128), tmQ, &ctl->q_full[s][qb], ka * 64, g * C::TM,
                    static_cast<int>(bh[s]));
      ++q_loads[s];
      return true;
    }
  };
  auto issue_k = [&](int s) -> bool {
#pragma unroll
    for (int b = 0; b < C::BPS; ++b) {
      const int jb = next_block(s);
      row0[s][b] = jb >= 0 ? jb * BS : a.N;  // N (out of range) pads with zeros
    }
    const uint32_t ks = k_loads % C::NKS;
    if (!wait_bounded(&ctl->k_empty[ks], ((k_loads / C::NKS) & 1) ^ 1, &ctl->abort)) return false;
    mbar_arrive_expect_tx(&ctl->k_full[ks], C::CH_BYTES);
#pragma unroll
    for (int b = 0; b < C::BPS; ++b)
#pragma unroll
      for (int ka = 0; ka < C::KATOMS; ++ka)
        tma_load_3d(smem + C::OFF_K + ks * C::CH_BYTES + ka * (C::NK * 128) + b * (BS * 128), tmK,
                    &ctl->k_full[ks], ka * 64, row0[s][b], static_cast<int>(bh[s]));
    ++k_loads;
    return true;
  };
  auto issue_v = [&](int s) -> bool {
    const uint32_t vs = v_loads % C::NVS;
    if (!wait_bounded(&ctl->v_empty[vs], ((v_loads / C::NVS) & 1) ^ 1, &ctl->abort)) return false;
    mbar_arrive_expect_tx(&ctl->v_full[vs], C::CH_BYTES);
#pragma unroll
    for (int b = 0; b < C::BPS; ++b)
#pragma unroll
      for (int ka = 0; ka < C::KATOMS; ++ka)
        tma_load_3d(smem + C::OFF_V + vs * C::CH_BYTES + ka * (C::NK * 128) + b * (BS * 128), tmV,
                    &ctl->v_full[vs], ka * 64, row0[s][b], static_cast<int>(bh[s]));
    ++v_loads;
    return true;
  };

  for (int s = 0; ok && s < kSlots; ++s) {
    ok = next_tile_of(s);
    if (ok && active[s]) ok = issue_k(s);
  }
  while (ok && (active[0] || active[1])) {
    for (int s = 0; ok && s < kSlots; ++s) {
      if (!active[s]) continue;
      ok = issue_v(s);
      if (!ok) break;
      if (j[s] == steps[s] - 1) {
        mbar_arrive(&ctl->t_empty[s][t[s] & 1]);
        ++t[s];
        ok = next_tile_of(s);
        if (ok && active[s]) ok = issue_k(s);
      } else {
        ++j[s];
        ok = issue_k(s);
      }
    }
  }
  if (ok) return;
  // On an early exit, let every copy already issued land before the CTA ends.
  for (int s = 0; s < kSlots; ++s)
    for (uint32_t b = 0; b < static_cast<uint32_t>(C::QB); ++b)
      if (q_loads[s] > b) {
        const uint32_t last = b + C::QB * ((q_loads[s] - 1 - b) / C::QB);
        wait_drain(&ctl->q_full[s][b], (last / C::QB) & 1);
      }
  for (uint32_t st = 0; st < static_cast<uint32_t>(C::NKS); ++st)
    if (k_loads > st) {
      const uint32_t last = st + C::NKS * ((k_loads - 1 - st) / C::NKS);
      wait_drain(&ctl->k_full[st], (last / C::NKS) & 1);
    }
  for (uint32_t st = 0; st < static_cast<uint32_t>(C::NVS); ++st)
    if (v_loads > st) {
      const uint32_t last = st + C::NVS * ((v_loads - 1 - st) / C::NVS);
      wait_drain(&ctl->v_full[st], (last / C::NVS) & 1);
    }
}

// ---------------------------------------------------------------- MMA issuer
// Order: S(0) of each slot, then per slot in turn O += P(j) V(j) and the
// slot's next S (step j+1 of its tile, or step 0 of its next tile).  MMAs of
// one thread complete in issue order, so a slot's next S overwrites S/P only
// after the P V that reads P, and the commit of a slot's S also reports that
// its previous P V has finished (the softmax relies on this to rescale O).
template <int BS, int D>
__device__ void mma_role(const FwdArgs& a, uint8_t* smem, Ctrl* ctl, uint32_t tmem) {
  using C = Cfg<BS, D>;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, C::NK, false, false);  // Q, K K-major
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);       // V MN-major
  const uint32_t q_base = smem_u32(smem + C::OFF_Q);
  const uint32_t k_base = smem_u32(smem + C::OFF_K);
  const uint32_t v_base = smem_u32(smem + C::OFF_V);
  uint32_t k_cons = 0, v_cons = 0;
  uint32_t q_uses[kSlots] = {0, 0}, p_seen[kSlots] = {0, 0};
  int t[kSlots] = {0, 0}, steps[kSlots] = {0, 0}, j[kSlots] = {0, 0};
  bool active[kSlots] = {true, true};
  bool ok = true;

  auto next_tile_of = [&](int s) -> bool {
    for (;;) {
      const int buf = t[s] & 1;
      if (!wait_bounded(&ctl->t_full[s][buf], (t[s] >> 1) & 1, &ctl->abort)) return false;
      const long long tile = ctl->info[s][buf].tile;
      const int n = ctl->info[s][buf].n;
      if (tile < 0) {
        active[s] = false;
        return true;
      }
      if (n == 0) {
        mbar_arrive(&ctl->t_empty[s][buf]);
        ++t[s];
        continue;
      }
      steps[s] = (n + C::BPS - 1) / C::BPS;
      j[s] = 0;
      return true;
    }
  };
  auto issue_qk = [&](int s) -> bool {
    const uint32_t qb = q_uses[s] % C::QB;
    if (j[s] == 0 &&
        !wait_bounded(&ctl->q_full[s][qb], (q_uses[s] / C::QB) & 1, &ctl->abort))
      return false;
    const uint32_t ks = k_cons % C::NKS;
    if (!wait_bounded(&ctl->k_full[ks], (k_cons / C::NKS) & 1, &ctl->abort)) return false;
    tc_fence_after();
    // Descriptors of consecutive K=16 slices differ only in the start
    // address field (address >> 4), so they are a base plus a constant.
    const uint64_t ad0 = sdesc_sw128(q_base + (s * C::QB + qb) * C::Q_BYTES, 16, 1024);
    const uint64_t bd0 = sdesc_sw128(k_base + ks * C::CH_BYTES, 16, 1024);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = ((kk >> 2) * (C::TM * 128) + (kk & 3) * 32) >> 4;  // TM == NK
      umma_bf16_ss(tmem + s * 128, ad0 + off, bd0 + off, kIdescQK, kk > 0 ? 1u : 0u);
    }
    umma_commit(&ctl->k_empty[ks]);
    umma_commit(&ctl->s_full[s]);
    if (j[s] == steps[s] - 1) {
      umma_commit(&ctl->q_empty[s][qb]);
      ++q_uses[s];
    }
    ++k_cons;
    return true;
  };
  auto issue_pv = [&](int s) -> bool {
    if (!wait_bounded(&ctl->p_full[s], p_seen[s] & 1, &ctl->abort)) return false;
    ++p_seen[s];
    const uint32_t vs = v_cons % C::NVS;
    if (!wait_bounded(&ctl->v_full[vs], (v_cons / C::NVS) & 1, &ctl->abort)) return false;
    tc_fence_after();
    const uint64_t bd0 = sdesc_sw128(v_base + vs * C::CH_BYTES, C::NK * 128, 1024);
    const uint32_t a0 = tmem + s * 128;
    const uint32_t d0 = tmem + C::TMEM_O + s * D;
#pragma unroll
    for (int kk = 0; kk < C::NK / 16; ++kk)  // P of keys 16kk..16kk+15: TMEM columns 8kk..8kk+7
      umma_bf16_ts(d0, a0 + kk * 8, bd0 + ((kk * 16 * 128) >> 4), kIdescPV,
                   (j[s] > 0 || kk > 0) ? 1u : 0u);
    umma_commit(&ctl->v_empty[vs]);
    ++v_cons;
    return true;
  };

  for (int s = 0; ok && s < kSlots; ++s) {
    ok = next_tile_of(s);
    if (ok && active[s]) ok = issue_qk(s);
  }
  while (ok && (active[0] || active[1])) {
    for (int s = 0; ok && s < kSlots; ++s) {
      if (!active[s]) continue;
      ok = issue_pv(s);
      if (!ok) break;
      if (j[s] == steps[s] - 1) {
        umma_commit(&ctl->o_full[s]);
        mbar_arrive(&ctl->t_empty[s][t[s] & 1]);
        ++t[s];
        ok = next_tile_of(s);
        if (ok && active[s]) ok = issue_qk(s);
      } else {
        ++j[s];
        ok = issue_qk(s);
      }
    }
  }
  // Every MMA issued must complete before the TMEM is released.
  umma_commit(&ctl->final_bar);
  wait_drain(&ctl->final_bar, 0);
}

// ------------------------------------------------------- softmax warpgroups
// Warpgroup s: thread i owns query row i of slot s's tile.  Per step it loads
// the scores of the blocks its row holds, takes the running maximum (the
// rescale of O is lazy: only when the maximum grows by more than 2^8), writes
// P over the first 64 score columns, and at the end of the tile stores
// O / l and the LSE.  Every TMEM access here waits for itself inside one asm
// statement (see sm100_ptx.cuh).
template <int BS, int D>
__device__ void softmax_role(int s, const FwdArgs& a, Ctrl* ctl, const uint32_t* bitmaps,
                             uint32_t tmem) {
  using C = Cfg<BS, D>;
  constexpr int GPB = BS / 32 < 1 ? 1 : BS / 32;  // 32-column groups per block
  const int wq = (threadIdx.x >> 5) & 3;         // TMEM lane quadrant
  const int lane = threadIdx.x & 31;
  const int row = wq * 32 + lane;                // query row of the tile
  const int sub = row / BS;                      // block row of the tile this thread belongs to
  const int qq = row % BS;                       // position inside that block row
  const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const uint32_t t_s = t_lane + s * 128;
  const uint32_t t_o = t_lane + C::TMEM_O + s * D;
  const float sl2 = a.scale_log2;
  constexpr float kNegInf = -INFINITY;
  const int W = a.W;
  uint32_t s_seen = 0, o_seen = 0;

  for (int t = 0;; ++t) {
    const int buf = t & 1;
    if (!warp_wait(&ctl->t_full[s][buf], (t >> 1) & 1, &ctl->abort)) return;
    const long long tile = ctl->info[s][buf].tile;
    const int n = ctl->info[s][buf].n;
    if (tile < 0) return;
    const uint32_t* bm = bitmaps + (s * 2 + buf) * bitmap_words<BS>(W);
    const int r_sub = static_cast<int>(tile % a.G) * C::R + sub;
    const bool row_ok = r_sub < a.M;

    float m_used = kNegInf;  // running maximum, log2 units of the scaled score
    float l = 0.f;           // running sum of 2^(x - m_used)
    const int steps = (n + C::BPS - 1) / C::BPS;
    BitIter it(bm + C::R * W, W);
    for (int j = 0; j < steps; ++j) {
      // 32-column groups of this step whose block this row holds, and those
      // of its diagonal block (both uniform over the warp).
      uint32_t own = 0, diag = 0;
#pragma unroll
      for (int b = 0; b < C::BPS; ++b) {
        const int jb = it.next();
        const uint32_t gm = ((1u << GPB) - 1u) << (b * GPB);
        if (row_ok && jb >= 0 && ((bm[sub * W + (jb >> 5)] >> (jb & 31)) & 1u)) own |= gm;
        if (a.causal && jb == r_sub) diag |= gm;
      }
      if (!warp_wait(&ctl->s_full[s], s_seen & 1, &ctl->abort)) return;
      ++s_seen;
      tc_fence_after();
      uint32_t u[128];
      tmem_ld128_groups_wait(t_s, own, u);

      // Scaled scores (log2 units), the causal mask, and the row maximum.
      float mx = kNegInf;
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) {
        if (!((own >> gi) & 1u)) continue;
        const bool dg = (diag >> gi) & 1u;
        float m0 = kNegInf, m1 = kNegInf;
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float x0 = __uint_as_float(u[gi * 32 + c]) * sl2;
          float x1 = __uint_as_float(u[gi * 32 + c + 1]) * sl2;
          if (dg) {  // key after the query (diagonal block only)
            const int kc = (gi * 32 + c) % BS;
            if (kc > qq) x0 = kNegInf;
            if (kc + 1 > qq) x1 = kNegInf;
          }
          u[gi * 32 + c] = __float_as_uint(x0);
          u[gi * 32 + c + 1] = __float_as_uint(x1);
          m0 = fmaxf(m0, x0);
          m1 = fmaxf(m1, x1);
        }
        mx = fmaxf(mx, fmaxf(m0, m1));
      }

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
      l *= factor;

      // P = 2^(x - m_used) in bf16 pairs over the first 64 score columns.
      const float mu = m_used == kNegInf ? 0.f : m_used;
      float r0 = 0.f, r1 = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) {
        if ((own >> gi) & 1u) {
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float p0 = ex2_approx(__uint_as_float(u[gi * 32 + c]) - mu);
            const float p1 = ex2_approx(__uint_as_float(u[gi * 32 + c + 1]) - mu);
            r0 += p0;
            r1 += p1;
            pk[gi * 16 + c / 2] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[gi * 16 + i] = 0u;
        }
      }
      l += r0 + r1;
      tmem_st64_wait(t_s, pk);
      // O holds the P V of every earlier step (this step's S being ready
      // means the previous P V has completed); bring it to the new maximum
      // before this step's P V adds to it.
      if (__any_sync(0xffffffffu, need_rescale)) {
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t w[32];
          tmem_ld32_wait(t_o + c0, w);
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * factor);
          tmem_st32_wait(t_o + c0, w);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full[s]);
    }

    // Epilogue: O / l in bf16 and LSE = (m + log2 l) ln 2, once the last P V
    // is done (an empty tile has no P V and stores O = 0, LSE = -inf).
    const long long bh = tile / a.G;
    const long long qtok = (tile - bh * a.G) * C::TM + row;
    uint4* orow = reinterpret_cast<uint4*>(a.O + (bh * a.N + qtok) * D);
    if (n > 0) {
      if (!warp_wait(&ctl->o_full[s], o_seen & 1, &ctl->abort)) return;
      ++o_seen;
      tc_fence_after();
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t w[32];
      if (n > 0) {
        tmem_ld32_wait(t_o + c0, w);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = 0u;
      }
      if (row_ok) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(w[q * 8 + 0]) * inv, __uint_as_float(w[q * 8 + 1]) * inv);
          v.y = pack_bf16x2(__uint_as_float(w[q * 8 + 2]) * inv, __uint_as_float(w[q * 8 + 3]) * inv);
          v.z = pack_bf16x2(__uint_as_float(w[q * 8 + 4]) * inv, __uint_as_float(w[q * 8 + 5]) * inv);
          v.w = pack_bf16x2(__uint_as_float(w[q * 8 + 6]) * inv, __uint_as_float(w[q * 8 + 7]) * inv);
          orow[c0 / 8 + q] = v;
        }
      }
    }
    if (row_ok)
      a.LSE[bh * a.N + qtok] = l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994531f : kNegInf;
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->t_empty[s][buf]);
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
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(ctl + 1);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(&ctl->t_full[s][b], 1);
        mbar_init(&ctl->t_empty[s][b], 4 + 2);  // the slot's softmax warps, the loader, the MMA issuer
        mbar_init(&ctl->q_full[s][b], 1);
        mbar_init(&ctl->q_empty[s][b], 1);
      }
      mbar_init(&ctl->s_full[s], 1);
      mbar_init(&ctl->p_full[s], 4);
      mbar_init(&ctl->o_full[s], 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&ctl->k_full[i], 1);
      mbar_init(&ctl->k_empty[i], 1);
      mbar_init(&ctl->v_full[i], 1);
      mbar_init(&ctl->v_empty[i], 1);
    }
    mbar_init(&ctl->final_bar, 1);
    ctl->abort.v = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  schedule<BS>(args, ctl);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  // Registers: the launch gives every thread kLaunchRegs; the softmax
  // warpgroups (a full score row per thread) take kSoftRegs, warpgroup 2
  // (the four single-warp roles) gives its share back.  Each warpgroup
  // executes its reallocation at one point, all four warps together.
  if (warp < 4 * kSlots) {
    reg_alloc_inc<kSoftRegs>();
  } else {
    reg_alloc_dec<kOtherRegs>();
  }
  if (warp < 4 * kSlots) {
    softmax_role<BS, D>(warp >> 2, args, ctl, bitmaps, tmem);
    __syncwarp();
  } else if (warp == kLoadWarp) {
    load_role<BS, D>(&tmQ, &tmK, &tmV, args, smem, ctl, bitmaps);
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if ((threadIdx.x & 31) == 0) mma_role<BS, D>(args, smem, ctl, tmem);
    __syncwarp();
  } else {
    build_role<BS, D>(warp - kBuildWarp, args, ctl, bitmaps);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace pp
}  // namespace bsa
