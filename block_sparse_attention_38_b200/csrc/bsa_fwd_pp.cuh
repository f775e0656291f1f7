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
// its own S, P and O in TMEM, its own Q/K/V stages in shared memory, its own
// producer warp and its own softmax warpgroup, in which thread i owns query
// row i of the tile (TMEM lane i): the row maximum and sum need no exchange
// between threads.  One MMA warp serves both slots without blocking on
// either: it polls each slot's barriers and issues whichever slot's next
// contraction is ready, so the tensor core works on one slot while the other
// slot's warpgroup turns scores into probabilities.  Roles (384 threads):
//   warps 0-3    softmax and epilogue of slot 0
//   warps 4-7    softmax and epilogue of slot 1
//   warps 8, 10  producer of slot 0 / slot 1: the slot's next tile from the
//                schedule, its block bitmaps from the CSR rows, and the TMA
//                loads of its Q, K, V (with an L2 prefetch of the next Q)
//   warp 9       tcgen05.mma issuer (and owner of the 512 TMEM columns)
//   warp 11      idle
//
// TMEM columns: S of slot s in [128 s, +128); P (bf16 pairs) over the first 64
// columns of S (d = 128) or in [256 + 64 s, +64) (d = 64); O after them.
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
constexpr int kProdWarp = 8;                // producer of slot s is warp kProdWarp + 2 s
constexpr int kMmaWarp = 9;
constexpr int kTiRing = 3;                  // tile-info entries per slot
// For d = 128, one group of 4 probabilities in kPolyEvery is computed by a
// polynomial on the FMA pipe instead of the MUFU ex2, to relieve the MUFU
// (measured: 947 -> 900 us on causal_loglinear_32k).  For d = 64 the steps
// have half the tensor work and the polynomial's extra instructions cost
// more than the MUFU time they save (727 -> 752 us on bernoulli_4k, 78 -> 82
// us on loglinear_4k), so every exponential there is an ex2.
#ifndef BSA_POLY_EVERY
#define BSA_POLY_EVERY 4
#endif
template <int D>
__host__ __device__ constexpr int poly_every() { return D == 64 ? 0 : BSA_POLY_EVERY; }

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
  static constexpr int KS = D == 64 ? 2 : 1;     // K stages per slot
  static constexpr int VS = KS;                  // V stages per slot
  static constexpr int SLOT_BYTES = QB * Q_BYTES + (KS + VS) * CH_BYTES;
  __host__ __device__ static constexpr int off_q(int s) { return s * SLOT_BYTES; }
  __host__ __device__ static constexpr int off_k(int s) { return s * SLOT_BYTES + QB * Q_BYTES; }
  __host__ __device__ static constexpr int off_v(int s) { return off_k(s) + KS * CH_BYTES; }
  static constexpr int OFF_CTRL = kSlots * SLOT_BYTES;
  static constexpr uint32_t TMEM_COLS = 512;
  // For d = 64, P of a slot has 64 TMEM columns of its own, so the slot's
  // next S can be computed while its P is still being written; for d = 128
  // there is no room, and P is written over the first 64 columns of S.
  static constexpr bool SEP_P = D == 64;
  static constexpr uint32_t TMEM_P = SEP_P ? 2 * 128 : 0;
  static constexpr uint32_t TMEM_O = SEP_P ? 2 * 128 + 2 * 64 : 2 * 128;  // O of slot s at TMEM_O + D s
  __host__ __device__ static constexpr uint32_t p_col(int s) { return SEP_P ? TMEM_P + 64 * s : 128 * s; }
  static_assert((Q_BYTES % 1024) == 0 && (CH_BYTES % 1024) == 0, "1024-byte aligned stages");
  static_assert(TMEM_O + kSlots * D <= TMEM_COLS, "TMEM layout");
  static_assert(TM == NK, "Q and K tiles share one slice-offset formula");
  static_assert(QB <= 2 && KS <= 2, "barrier arrays");
};

constexpr int kMaxChunks = 64;               // chunks one tile may be cut into
constexpr int kCutShares = 2;                // a tile is cut when it costs more than this many slot shares

// The plan every CTA computes identically (see `schedule`).
struct Plan {
  long long n_light;                // light tiles in all
  long long kt;                     // heavy tiles in all
  long long kh;                     // heavy work units in all (a cut tile counts once per chunk)
  long long scan[kWarps];
  int skip;                         // rounds of light tiles a slot holding a heavy unit sits out
  int kg;                           // heavy groups per batch element
  int kc;                           // heavy units per batch element
  int heavy_hg[kMaxHeavyGroups];    // heavy groups of one batch element, in order
  int heavy_pre[kMaxHeavyGroups + 1];  // heavy units before heavy group j (prefix of chunk counts)
  int heavy_cs[kMaxHeavyGroups];    // group cost while planning; then steps per chunk
};

// One work unit: a tile, or one chunk of the key walk of a cut tile.
struct Unit {
  long long tile;                   // -1: no more work for this slot
  int lo;                           // first step of the walk
  int len;                          // steps at most (the last chunk takes all that remain)
  int nch;                          // chunks of the tile (1: not cut)
  int part;                         // workspace slot of this chunk; its tile's chunks are
                                    // the slots part - c .. part - c + nch - 1
  int c;                            // chunk index
};

// One slot's position in the plan (its producer warp advances it).
struct Cursor {
  long long heavy[2];               // this slot's heavy units
  long long round;                  // next round of light tiles
  long long hp;                     // heavy tiles known to lie before the current light tile
  int n_heavy;
  int next_heavy;
};

struct TileInfo {
  long long tile;  // tile index, -1 = no more work for this slot
  int n;           // union size in blocks
  int lo, cnt;     // this unit's steps: lo .. lo + cnt - 1 of the walk
  int nch, part, c;  // see Unit
};

// The barriers of one slot.
struct SlotBars {
  uint64_t t_full[kTiRing], t_empty[kTiRing];  // tile-info ring
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full, p_full, o_full;
  uint64_t s_free, pv_done;                    // separate-P layout only
};

struct Ctrl {
  SlotBars sb[kSlots];
  uint64_t final_bar;
  TileInfo info[kSlots][kTiRing];
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
//     2V heavy tiles.  With more than V of them the costs are too even for
//     the steps below to pay, and every tile is treated as light.
//  2. A heavy tile that costs more than kCutShares whole shares (2 thr each)
//     is cut into chunks of about one share along its key walk ("split long
//     rows into kv-chunks"), when the caller gave a workspace for the partial
//     results and the chunks fit in it and in V (else chunks are made longer).
//  3. The heavy units (uncut heavy tiles and chunks) go first, unit k to slot
//     k mod V; the light tiles, in tile order, are dealt out in rounds of one
//     tile per slot, the slots holding a heavy unit sitting out the first
//     `skip` rounds, skip = average heavy unit cost / average light cost.
template <int BS>
__device__ void schedule(const FwdArgs& a, Ctrl* ctl) {
  constexpr int BPS = 128 / BS;
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
    const long long cst = group_cost<BS>(a, hg);
    if (cst > thr) {
      pl.heavy_hg[hexcl] = static_cast<int>(hg);
      pl.heavy_cs[hexcl] = static_cast<int>(min(cst, 0x7fffffffLL));
      ++hexcl;
    }
  }
  __syncthreads();  // every thread's heavy groups are written before thread 0 deals them out
  if (tid == 0) {
    if (Kg * nb > V) Kg = 0;
    // Chunk counts: a group of cost c > kCutShares shares (2 thr each) is cut
    // into ceil(c / (2 f thr)) chunks, f = 1, 2, 4, ... until all units fit in
    // V and in the workspace.  (A tile only a little above one share is left
    // whole: there the cut's own costs, the partial results' round trip and
    // the chunks' concurrent start, outweigh the balance it buys.)
    const long long cap = min(V, static_cast<long long>(a.part_cap));
    const long long cut_above = kCutShares * 2 * thr;
    long long Kc = Kg;
    for (long long f = 1; Kg > 0 && cap > 0 && thr > 0; f *= 2) {
      const long long unit = 2 * f * thr;
      long long kc = 0;
      for (long long j = 0; j < Kg; ++j) {
        const long long cst = pl.heavy_cs[j];
        kc += cst > cut_above ? min(static_cast<long long>(kMaxChunks), (cst + unit - 1) / unit) : 1;
      }
      if (kc * nb <= cap || kc == Kg) {
        Kc = 0;
        for (long long j = 0; j < Kg; ++j) {
          const long long cst = pl.heavy_cs[j];
          const long long nch =
              cst > cut_above ? min(static_cast<long long>(kMaxChunks), (cst + unit - 1) / unit) : 1;
          const long long steps = (cst + BPS - 1) / BPS;  // estimated steps of the walk
          pl.heavy_pre[j] = static_cast<int>(Kc);
          pl.heavy_cs[j] = static_cast<int>((steps + nch - 1) / nch);
          Kc += nch;
        }
        break;
      }
    }
    if (Kc == Kg) {  // nothing cut
      for (long long j = 0; j < Kg; ++j) {
        pl.heavy_pre[j] = static_cast<int>(j);
        pl.heavy_cs[j] = 0x7fffffff;
      }
    }
    pl.heavy_pre[Kg] = static_cast<int>(Kc);
    const long long Kt = Kg * nb;  // heavy tiles
    const long long Kh = Kc * nb;  // heavy units, <= V
    const long long n_light = a.num_tiles - Kt;
    long long skip = 0;
    if (Kh > 0 && n_light > 0 && V - Kh > 0) {
      const double heavy_avg = static_cast<double>(Hper * nb) / Kh;
      const double light_avg = static_cast<double>(total - Hper * nb) / n_light;
      skip = static_cast<long long>(heavy_avg / light_avg + 0.5);
      const long long most = n_light / (V - Kh);
      if (skip > most) skip = most;
    }
    pl.kt = Kt;
    pl.kh = Kh;
    pl.kg = static_cast<int>(Kg);
    pl.kc = static_cast<int>(Kc);
    pl.n_light = n_light;
    pl.skip = static_cast<int>(skip);
    for (int s = 0; s < kSlots; ++s) {
      Cursor& cu = ctl->cur[s];
      const long long v = static_cast<long long>(kSlots) * blockIdx.x + s;
      int nh = 0;
      for (long long k = v; k < Kh && nh < 2; k += V) cu.heavy[nh++] = k;
      cu.n_heavy = nh;
      cu.next_heavy = 0;
      cu.round = 0;
      cu.hp = 0;
    }
  }
  __syncthreads();
}

// Heavy unit k of the plan: its tile and its chunk.
__device__ __forceinline__ Unit heavy_unit(const FwdArgs& a, const Plan& pl, long long k) {
  const long long HG = static_cast<long long>(a.H) * a.G;
  const long long b = k / pl.kc;
  const int r = static_cast<int>(k - b * pl.kc);
  int lo = 0, hi = pl.kg - 1;  // the group j with heavy_pre[j] <= r < heavy_pre[j + 1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pl.heavy_pre[mid] <= r) lo = mid; else hi = mid - 1;
  }
  Unit u;
  u.tile = b * HG + pl.heavy_hg[lo];
  u.nch = pl.heavy_pre[lo + 1] - pl.heavy_pre[lo];
  u.c = r - pl.heavy_pre[lo];
  u.lo = u.nch > 1 ? u.c * pl.heavy_cs[lo] : 0;
  u.len = u.c < u.nch - 1 ? pl.heavy_cs[lo] : 0x7fffffff;
  u.part = static_cast<int>(k);
  return u;
}

// Next unit of slot worker v (one builder lane), tile -1 when none is left:
// its heavy units first, then its light tiles in increasing order.
__device__ __forceinline__ Unit next_unit(const FwdArgs& a, const Plan& pl, Cursor& cu, long long v) {
  if (cu.next_heavy < cu.n_heavy) return heavy_unit(a, pl, cu.heavy[cu.next_heavy++]);
  Unit u;
  u.tile = -1;
  u.lo = 0;
  u.len = 0x7fffffff;
  u.nch = 1;
  u.part = 0;
  u.c = 0;
  const long long V = static_cast<long long>(kSlots) * gridDim.x;
  const long long Kh = pl.kh;
  const bool skipping = pl.skip > 0;             // slots 0 .. Kh-1 hold a heavy unit
  const long long others = V - Kh;               // slots without one
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
  if (i >= pl.n_light) return u;
  // Light tile i is tile i + (heavy tiles before it); the heavy tiles are in
  // increasing tile order and i only grows, so the count is kept across calls.
  const long long HG = static_cast<long long>(a.H) * a.G;
  long long t = i + cu.hp;
  while (cu.hp < pl.kt && (cu.hp / pl.kg) * HG + pl.heavy_hg[cu.hp % pl.kg] <= t) {
    ++cu.hp;
    t = i + cu.hp;
  }
  u.tile = t;
  return u;
}

// ---------------------------------------------------------- producer warps
// Warp kProdWarp + 2s, for slot s: take the slot's next tile from the
// schedule, turn its CSR rows into the R block-row bitmaps and their union
// (all lanes), publish it in the slot's tile-info ring, and issue (lane 0)
// the TMA loads of its Q and, step by step, K and V into the slot's stages.
// The tile after it is looked up at the same time and its Q prefetched into L2.
template <int BS, int D>
__device__ void produce_role(int s, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                             const CUtensorMap* tmV, const FwdArgs& a, uint8_t* smem, Ctrl* ctl,
                             uint32_t* bitmaps) {
  using C = Cfg<BS, D>;
  const int lane = threadIdx.x & 31;
  const int W = a.W;
  const int BMW = bitmap_words<BS>(W);
  const long long v = static_cast<long long>(kSlots) * blockIdx.x + s;
  SlotBars& B = ctl->sb[s];
  uint32_t q_loads = 0, k_loads = 0, v_loads = 0;
  Unit peeked;            // lane 0: the slot's next unit, once looked up
  bool have_peek = false;
  bool ok = true;
  if (lane == 0) {
    prefetch_tensormap(tmQ);
    prefetch_tensormap(tmK);
    prefetch_tensormap(tmV);
  }
  for (int t = 0;; ++t) {
    const int buf = t % kTiRing;
    int w_ok = 1;
    Unit u;
    u.tile = -1;
    if (lane == 0) {
      w_ok = wait_bounded(&B.t_empty[buf], ((t / kTiRing) & 1) ^ 1, &ctl->abort);
      if (w_ok) {
        u = have_peek ? peeked : next_unit(a, ctl->plan, ctl->cur[s], v);
        if (u.tile >= 0) {
          peeked = next_unit(a, ctl->plan, ctl->cur[s], v);
        } else {
          peeked.tile = -1;
        }
        have_peek = true;
        if (peeked.tile >= 0) {  // the next unit's Q into L2
          const long long pbh = peeked.tile / a.G;
          const int pg = static_cast<int>(peeked.tile - pbh * a.G);
#pragma unroll
          for (int ka = 0; ka < C::KATOMS; ++ka)
            tma_prefetch_3d(tmQ, ka * 64, pg * C::TM, static_cast<int>(pbh));
        }
      }
    }
    if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
    const long long tile = __shfl_sync(0xffffffffu, u.tile, 0);
    uint32_t* bm = bitmaps + (s * kTiRing + buf) * BMW;
    int n = 0;
    long long bh = 0;
    int g = 0;
    if (tile >= 0) {
      for (int w = lane; w < BMW; w += 32) bm[w] = 0u;
      __syncwarp();
      bh = tile / a.G;
      g = static_cast<int>(tile - bh * a.G);
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
    // This unit's part of the walk.
    const int all_steps = (n + C::BPS - 1) / C::BPS;
    int lo = 0, cnt = 0;
    if (lane == 0 && tile >= 0) {
      lo = min(u.lo, all_steps);
      cnt = min(u.len, all_steps - lo);
      TileInfo& ti = ctl->info[s][buf];
      ti.lo = lo;
      ti.cnt = cnt;
      ti.nch = u.nch;
      ti.part = u.part;
      ti.c = u.c;
    }
    if (lane == 0) {
      ctl->info[s][buf].tile = tile;
      ctl->info[s][buf].n = n;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&B.t_full[buf]);
    if (tile < 0) break;
    if (lane == 0) {
      if (cnt > 0) {
        const uint32_t qb = q_loads % C::QB;
        ok = wait_bounded(&B.q_empty[qb], ((q_loads / C::QB) & 1) ^ 1, &ctl->abort);
        if (ok) {
          mbar_arrive_expect_tx(&B.q_full[qb], C::Q_BYTES);
#pragma unroll
          for (int ka = 0; ka < C::KATOMS; ++ka)
            tma_load_3d(smem + C::off_q(s) + qb * C::Q_BYTES + ka * (C::TM * 128), tmQ, &B.q_full[qb],
                        ka * 64, g * C::TM, static_cast<int>(bh));
          ++q_loads;
        }
        BitIter it(bm + C::R * W, W);
        it.skip(lo * C::BPS);
        for (int j = 0; ok && j < cnt; ++j) {
          int row0[C::BPS];  // first token of each block of the step; N (out of range) pads
#pragma unroll
          for (int b = 0; b < C::BPS; ++b) {
            const int jb = it.next();
            row0[b] = jb >= 0 ? jb * BS : a.N;
          }
          const uint32_t ks = k_loads % C::KS;
          ok = wait_bounded(&B.k_empty[ks], ((k_loads / C::KS) & 1) ^ 1, &ctl->abort);
          if (!ok) break;
          mbar_arrive_expect_tx(&B.k_full[ks], C::CH_BYTES);
#pragma unroll
          for (int b = 0; b < C::BPS; ++b)
#pragma unroll
            for (int ka = 0; ka < C::KATOMS; ++ka)
              tma_load_3d(smem + C::off_k(s) + ks * C::CH_BYTES + ka * (C::NK * 128) + b * (BS * 128),
                          tmK, &B.k_full[ks], ka * 64, row0[b], static_cast<int>(bh));
          ++k_loads;
          const uint32_t vs = v_loads % C::VS;
          ok = wait_bounded(&B.v_empty[vs], ((v_loads / C::VS) & 1) ^ 1, &ctl->abort);
          if (!ok) break;
          mbar_arrive_expect_tx(&B.v_full[vs], C::CH_BYTES);
#pragma unroll
          for (int b = 0; b < C::BPS; ++b)
#pragma unroll
            for (int ka = 0; ka < C::KATOMS; ++ka)
              tma_load_3d(smem + C::off_v(s) + vs * C::CH_BYTES + ka * (C::NK * 128) + b * (BS * 128),
                          tmV, &B.v_full[vs], ka * 64, row0[b], static_cast<int>(bh));
          ++v_loads;
        }
      }
      if (ok) mbar_arrive(&B.t_empty[buf]);  // the producer is done with this tile's bitmaps
    }
    if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { ok = false; break; }
  }
  if (ok || lane != 0) return;
  // On an early exit, let every copy already issued land before the CTA ends.
  for (uint32_t b = 0; b < static_cast<uint32_t>(C::QB); ++b)
    if (q_loads > b) {
      const uint32_t last = b + C::QB * ((q_loads - 1 - b) / C::QB);
      wait_drain(&B.q_full[b], (last / C::QB) & 1);
    }
  for (uint32_t st = 0; st < static_cast<uint32_t>(C::KS); ++st)
    if (k_loads > st) {
      const uint32_t last = st + C::KS * ((k_loads - 1 - st) / C::KS);
      wait_drain(&B.k_full[st], (last / C::KS) & 1);
    }
  for (uint32_t st = 0; st < static_cast<uint32_t>(C::VS); ++st)
    if (v_loads > st) {
      const uint32_t last = st + C::VS * ((v_loads - 1 - st) / C::VS);
      wait_drain(&B.v_full[st], (last / C::VS) & 1);
    }
}

// ---------------------------------------------------------------- MMA issuer
// One thread serves both slots without blocking on either: each pass it
// tries, per slot, the next O += P V and the next S = Q K^T, and issues those
// whose barriers have completed (non-blocking tests).  Per slot, S of step
// g+1 runs at most one step ahead of the P V of step g.  With P written over
// S, a slot's next S is issued only after its P V; MMAs of one thread
// complete in issue order, so S overwrites P only after the P V has read it,
// and the commit of S also reports that the previous P V has finished.  With
// P in its own columns, a slot's next S waits only until the softmax has
// loaded the current scores (s_free), and each P V commits pv_done.
struct PStep {          // a step whose S is issued and whose P V is not
  int buf;
  bool first, last;
};

struct MmaSlot {        // the MMA issuer's state for one slot (kept in registers)
  int t = 0;            // tile-info entry of the S side's tile
  int qsteps = 0, qj = 0;  // steps of that tile, next S step (qj == qsteps: next tile)
  bool done = false;    // the S side has seen the end of the slot's work
  uint32_t q_uses = 0, k_cons = 0, v_cons = 0, qk_issued = 0, p_seen = 0;
  PStep front, back;    // P V queue (at most two steps)
  int pcount = 0;
};

template <int BS, int D>
__device__ void mma_role(const FwdArgs& a, uint8_t* smem, Ctrl* ctl, uint32_t tmem) {
  using C = Cfg<BS, D>;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, C::NK, false, false);  // Q, K K-major
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);       // V MN-major
  const uint32_t sbase = smem_u32(smem);
  MmaSlot sl0, sl1;

  // Next S = Q K^T of slot s, if every input is ready: 1 issued (or an empty
  // tile skipped), 0 not ready, -1 inconsistent tile info.
  auto try_qk = [&](MmaSlot& st, int s) -> int {
    SlotBars& B = ctl->sb[s];
    if (st.done) return 0;
    if (st.qj == st.qsteps) {  // the next tile
      const int buf = st.t % kTiRing;
      if (!mbar_test_wait(&B.t_full[buf], (st.t / kTiRing) & 1)) return 0;
      const long long tile = ctl->info[s][buf].tile;
      const int n = ctl->info[s][buf].n;
      if (tile < 0) {
        st.done = true;
        return 0;
      }
      const int cnt = ctl->info[s][buf].cnt;
      if (tile >= a.num_tiles || n > a.M || cnt < 0 || cnt > n) return -1;  // never for a consistent schedule
      if (cnt == 0) {
        mbar_arrive(&B.t_empty[buf]);
        ++st.t;
        return 1;
      }
      st.qsteps = cnt;
      st.qj = 0;
    }
    if (!C::SEP_P && st.pcount > 0) return 0;  // P lives in S: its P V goes first
    const uint32_t qb = st.q_uses % C::QB;
    if (st.qj == 0 && !mbar_test_wait(&B.q_full[qb], (st.q_uses / C::QB) & 1)) return 0;
    if (C::SEP_P && st.qk_issued > 0 && !mbar_test_wait(&B.s_free, (st.qk_issued - 1) & 1))
      return 0;
    const uint32_t ks = st.k_cons % C::KS;
    if (!mbar_test_wait(&B.k_full[ks], (st.k_cons / C::KS) & 1)) return 0;
    tc_fence_after();
    const uint64_t ad = sdesc_sw128(sbase + C::off_q(s) + qb * C::Q_BYTES, 16, 1024);
    const uint64_t bd = sdesc_sw128(sbase + C::off_k(s) + ks * C::CH_BYTES, 16, 1024);
    umma_qk_chain<D / 16>(tmem + s * 128, static_cast<uint32_t>(ad), static_cast<uint32_t>(ad >> 32),
                          static_cast<uint32_t>(bd), static_cast<uint32_t>(bd >> 32), kIdescQK);
    umma_commit(&B.k_empty[ks]);
    umma_commit(&B.s_full);
    PStep e;
    e.buf = st.t % kTiRing;
    e.first = st.qj == 0;
    e.last = st.qj == st.qsteps - 1;
    if (e.last) {
      umma_commit(&B.q_empty[qb]);
      ++st.q_uses;
      ++st.t;
    }
    ++st.qj;
    ++st.k_cons;
    ++st.qk_issued;
    if (st.pcount == 0) st.front = e; else st.back = e;
    ++st.pcount;
    return 1;
  };
  // Next O += P V of slot s, if its P and V are ready.
  auto try_pv = [&](MmaSlot& st, int s) -> int {
    SlotBars& B = ctl->sb[s];
    if (st.pcount == 0) return 0;
    if (!mbar_test_wait(&B.p_full, st.p_seen & 1)) return 0;
    const uint32_t vs = st.v_cons % C::VS;
    if (!mbar_test_wait(&B.v_full[vs], (st.v_cons / C::VS) & 1)) return 0;
    tc_fence_after();
    const PStep e = st.front;
    // P of keys 16kk..16kk+15 sits in TMEM columns p_col + 8kk .. +7.
    const uint64_t bd = sdesc_sw128(sbase + C::off_v(s) + vs * C::CH_BYTES, C::NK * 128, 1024);
    umma_pv_chain8(tmem + C::TMEM_O + s * D, tmem + C::p_col(s), static_cast<uint32_t>(bd),
                   static_cast<uint32_t>(bd >> 32), kIdescPV, e.first ? 0u : 1u);
    umma_commit(&B.v_empty[vs]);
    if (C::SEP_P) umma_commit(&B.pv_done);
    if (e.last) {
      umma_commit(&B.o_full);
      mbar_arrive(&B.t_empty[e.buf]);
    }
    ++st.p_seen;
    ++st.v_cons;
    st.front = st.back;
    --st.pcount;
    return 1;
  };

  long long idle_since = clock64();
  int oldest = 0;  // the slot whose pending P V was queued first
  while (!(sl0.done && sl0.pcount == 0 && sl1.done && sl1.pcount == 0)) {
    const int r0 = try_pv(sl0, 0), r1 = try_qk(sl0, 0);
    const int r2 = try_pv(sl1, 1), r3 = try_qk(sl1, 1);
    if (r0) oldest = 1;
    if (r2) oldest = 0;
    if (r1 < 0 || r3 < 0) {
      atomicOr(&g_status, BSA_STATUS_INTERNAL);
      ctl->abort.v = 1;
      break;
    }
    if (r0 | r1 | r2 | r3) {
      idle_since = clock64();
    } else {
      if (ctl->abort.v) break;
      // Nothing is ready: sleep in the barrier the issuer most likely waits
      // for (a slot's P, its softmax warps being the usual hold-up), which
      // leaves this sub-partition's issue slots to the softmax warps.
      int ws = oldest;
      if ((ws == 0 ? sl0.pcount : sl1.pcount) == 0) ws ^= 1;
      const MmaSlot& w = ws == 0 ? sl0 : sl1;
      if (w.pcount > 0)
        mbar_try_wait_hint(&ctl->sb[ws].p_full, w.p_seen & 1, 2000);
      else
        __nanosleep(64);
      if (clock64() - idle_since > kWaitLimitCycles) {
        atomicOr(&g_status, BSA_STATUS_TIMEOUT);
        ctl->abort.v = 1;
        break;
      }
    }
  }
  // Every MMA issued must complete before the TMEM is released.
  umma_commit(&ctl->final_bar);
  wait_drain(&ctl->final_bar, 0);
}

// ------------------------------------------------------------ chunk merge
// Arrival of one warp's chunk at its tile's count word (epoch << 8 | count):
// a word from an earlier launch counts as zero.  Returns the count with this
// arrival included.
__device__ __forceinline__ int chunk_arrive(unsigned long long* word, unsigned long long epoch) {
  unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(word);
  for (;;) {
    const unsigned long long nv = (old >> 8) == epoch ? old + 1ull : (epoch << 8) | 1ull;
    const unsigned long long seen = atomicCAS(word, old, nv);
    if (seen == old) return static_cast<int>(nv & 0xffull);
    old = seen;
  }
}

// Epilogue of one chunk of a cut tile, per warp (its 32 query rows): store
// the chunk's O (still multiplied by l) and its (m, l); the warp whose arrival
// completes the count of its quadrant merges the tile's chunks in chunk
// order, O = sum_c 2^(m_c - M) O_c / L and LSE = (M + log2 L) ln 2 with
// M = max_c m_c and L = sum_c 2^(m_c - M) l_c over the chunks holding keys
// of the row -- the same softmax over the union of the chunks' keys ("Block
// Sparse Attention with Log-Linear Complexity", section 3.3).  Every chunk,
// its own included, is read back from the workspace, so the result does not
// depend on which chunk finishes last.
template <int D>
__device__ __forceinline__ void chunk_epilogue(const FwdArgs& a, const TileInfo& ti, uint32_t t_o,
                                               float m_used, float l, int row, int wq, bool row_ok,
                                               uint4* orow, float* lse) {
  const int lane = threadIdx.x & 31;
  const int part = ti.part, base = ti.part - ti.c, nch = ti.nch;
  const bool have_o = ti.cnt > 0;  // uniform over the warp
  float* po = a.part_o + static_cast<long long>(part) * D * 128 + row;
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t w[32];
    if (have_o) {
      __syncwarp();
      tmem_ld32_wait(t_o + c0, w);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) w[i] = 0u;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) __stcg(po + (c0 + i) * 128, __uint_as_float(w[i]));
  }
  __stcg(a.part_ml + static_cast<long long>(part) * 128 + row, make_float2(m_used, l));
  __threadfence();
  __syncwarp();
  int last = 0;
  if (lane == 0) last = chunk_arrive(a.part_cnt + static_cast<long long>(base) * 4 + wq, a.epoch) == nch;
  if (!__shfl_sync(0xffffffffu, last, 0)) return;
  __threadfence();

  const float2* ml0 = a.part_ml + static_cast<long long>(base) * 128 + row;
  float M = -INFINITY;
  for (int cc = 0; cc < nch; ++cc) {
    const float2 ml = __ldcg(ml0 + cc * 128);
    if (ml.y > 0.f) M = fmaxf(M, ml.x);
  }
  float L = 0.f;
  for (int cc = 0; cc < nch; ++cc) {
    const float2 ml = __ldcg(ml0 + cc * 128);
    if (ml.y > 0.f) L += ml.y * ex2_approx(ml.x - M);
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const float* pb = a.part_o + static_cast<long long>(base) * D * 128 + row;
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 32) {
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
#pragma unroll 1
    for (int cc = 0; cc < nch; ++cc) {
      const float2 ml = __ldcg(ml0 + cc * 128);
      const float wt = ml.y > 0.f ? ex2_approx(ml.x - M) * inv : 0.f;
      const float* pc = pb + static_cast<long long>(cc) * D * 128 + c0 * 128;
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = fmaf(wt, __ldcg(pc + i * 128), acc[i]);
    }
    if (row_ok) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 v;
        v.x = pack_bf16x2(acc[q * 8 + 0], acc[q * 8 + 1]);
        v.y = pack_bf16x2(acc[q * 8 + 2], acc[q * 8 + 3]);
        v.z = pack_bf16x2(acc[q * 8 + 4], acc[q * 8 + 5]);
        v.w = pack_bf16x2(acc[q * 8 + 6], acc[q * 8 + 7]);
        orow[c0 / 8 + q] = v;
      }
    }
  }
  if (row_ok) *lse = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
}

// ------------------------------------------------------- softmax warpgroups
// Warpgroup s: thread i owns query row i of slot s's tile.  A step is taken
// in two halves of 64 score columns: load the blocks the row holds, scale,
// mask the diagonal block of a causal tile, and keep a running maximum; the
// rescale is lazy (only when the maximum grows by more than 2^8), and when
// the second half raises it, the first half's P is rescaled in place.  P (bf16
// pairs) goes to the slot's P columns; at the end of the tile O / l and the
// LSE are stored.  Every TMEM access here waits for itself inside one asm
// statement (see sm100_ptx.cuh).
template <int BS, int D, bool POS, bool CAUSAL>
__device__ void softmax_role(int s, const FwdArgs& a, Ctrl* ctl, const uint32_t* bitmaps,
                             uint32_t tmem) {
  using C = Cfg<BS, D>;
  constexpr int GPB = BS / 32;                   // 32-column groups per block
  const int wq = (threadIdx.x >> 5) & 3;         // TMEM lane quadrant
  const int lane = threadIdx.x & 31;
  const int row = wq * 32 + lane;                // query row of the tile
  const int sub = row / BS;                      // block row of the tile this thread belongs to
  const int qq = row % BS;                       // position inside that block row
  const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const uint32_t t_s = t_lane + s * 128;
  const uint32_t t_p = t_lane + C::p_col(s);
  const uint32_t t_o = t_lane + C::TMEM_O + s * D;
  const float sl2 = a.scale_log2;
  constexpr float kNegInf = -INFINITY;
  const int W = a.W;
  SlotBars& B = ctl->sb[s];
  uint32_t s_seen = 0, o_seen = 0;

  for (int t = 0;; ++t) {
    const int buf = t % kTiRing;
    if (!warp_wait(&B.t_full[buf], (t / kTiRing) & 1, &ctl->abort)) return;
    const long long tile = ctl->info[s][buf].tile;
    const int n = ctl->info[s][buf].n;
    if (tile < 0) return;
    const TileInfo& ti = ctl->info[s][buf];  // in shared memory until the t_empty arrival
    if (tile >= a.num_tiles || n > a.M || ti.cnt < 0 || ti.cnt > n ||
        (ti.nch > 1 && (ti.part < ti.c || ti.part - ti.c + ti.nch > a.part_cap))) {  // never for a consistent schedule
      if (lane == 0) {
        atomicOr(&g_status, BSA_STATUS_INTERNAL);
        ctl->abort.v = 1;
      }
      return;
    }
    const uint32_t* bm = bitmaps + (s * kTiRing + buf) * bitmap_words<BS>(W);
    const int r_sub = static_cast<int>(tile % a.G) * C::R + sub;
    const bool row_ok = r_sub < a.M;

    float m_used = kNegInf;  // running maximum, log2 units of the scaled score
    float l = 0.f;           // running sum of 2^(x - m_used)
    BitIter it(bm + C::R * W, W);
    it.skip(ti.lo * C::BPS);
    for (int j = 0; j < ti.cnt; ++j) {
      // 32-column groups of this step whose block this row holds, and those
      // of its diagonal block (both uniform over the warp).
      uint32_t own = 0, diag = 0;
#pragma unroll
      for (int b = 0; b < C::BPS; ++b) {
        const int jb = it.next();
        const uint32_t gm = ((1u << GPB) - 1u) << (b * GPB);
        if (row_ok && jb >= 0 && ((bm[sub * W + (jb >> 5)] >> (jb & 31)) & 1u)) own |= gm;
        if (CAUSAL && jb == r_sub) diag |= gm;  // CAUSAL: a template parameter equal to a.causal
      }
      diag &= own;
      if (!warp_wait(&B.s_full, s_seen & 1, &ctl->abort)) return;
      const uint32_t g_step = s_seen++;        // steps of this slot before this one
      tc_fence_after();
      float osc = 1.f;                         // factor O must take before this step's P V
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const uint32_t ho = (own >> (2 * h)) & 3u, hd = (diag >> (2 * h)) & 3u;
        float x[64];
        __syncwarp();
        if (ho == 3u) {
          tmem_ld64_wait(t_s + 64 * h, x);
        } else if (ho == 1u) {
          tmem_ld32lo_wait(t_s + 64 * h, x);
        } else if (ho == 2u) {
          tmem_ld32hi_wait(t_s + 64 * h + 32, x);
        }
        if (C::SEP_P && h == 1) {              // the scores are in registers: S may be rewritten
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&B.s_free);
        }
        // Row maximum of the scaled scores, taken on the raw scores (their
        // minimum for a negative scale); on the diagonal block of a causal
        // tile, keys after the query are first set to the value that scales
        // to -inf.
        constexpr bool pos = POS;                // the scale's sign, a template parameter
        const float sentinel = pos ? kNegInf : INFINITY;
        float hraw = sentinel;
#pragma unroll
        for (int gi = 0; gi < 2; ++gi) {
          if (!((ho >> gi) & 1u)) continue;
          if ((hd >> gi) & 1u) {               // keys after the query (diagonal block only)
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if ((64 * h + gi * 32 + c) % BS > qq) x[gi * 32 + c] = sentinel;
          }
          float ma = sentinel, mb = sentinel;
          if constexpr (pos) {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              ma = max3f(ma, x[gi * 32 + c], x[gi * 32 + c + 1]);
              mb = max3f(mb, x[gi * 32 + c + 2], x[gi * 32 + c + 3]);
            }
            hraw = max3f(hraw, ma, mb);
          } else {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              ma = min3f(ma, x[gi * 32 + c], x[gi * 32 + c + 1]);
              mb = min3f(mb, x[gi * 32 + c + 2], x[gi * 32 + c + 3]);
            }
            hraw = min3f(hraw, ma, mb);
          }
        }
        const float hm = hraw * sl2;           // -inf when no key of the half is held
        // Lazy rescale: the running maximum moves only when it is exceeded by
        // more than the threshold (P stays <= 2^8 otherwise).
        const bool need = hm > m_used + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          float f = 1.f;
          if (need) {
            if (m_used != kNegInf) f = ex2_approx(m_used - hm);
            m_used = hm;
          }
          l *= f;
          osc *= f;
          if (h == 1 && __any_sync(0xffffffffu, f != 1.f)) {
            // The first half's P was taken against the old maximum.
            uint32_t w[32];
            __syncwarp();
            tmem_ld32_wait(t_p, w);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float lo = __uint_as_float(w[i] << 16) * f;
              const float hi = __uint_as_float(w[i] & 0xffff0000u) * f;
              w[i] = pack_bf16x2(lo, hi);
            }
            tmem_st32_wait(t_p, w);
          }
        }
        // P = 2^(x - m_used) in bf16 pairs: keys 64h .. 64h+63 to P columns 32h .. 32h+31.
        const float nmu = m_used == kNegInf ? 0.f : -m_used;
        float sa = 0.f, sb = 0.f, sc = 0.f, sd = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int gi = 0; gi < 2; ++gi) {
          if ((ho >> gi) & 1u) {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              float d0 = x[gi * 32 + c], d1 = x[gi * 32 + c + 1];
              float d2 = x[gi * 32 + c + 2], d3 = x[gi * 32 + c + 3];
              fma2(d0, d1, sl2, nmu);              // scaled score minus the maximum
              fma2(d2, d3, sl2, nmu);
              float p0, p1, p2, p3;
              constexpr int kPoly = poly_every<D>();
              if (kPoly > 0 && (c / 4) % (kPoly > 0 ? kPoly : 1) == kPoly - 1) {
                exp2_poly2(d0, d1);                // this share of 2^x on the FMA pipe
                exp2_poly2(d2, d3);
                p0 = d0; p1 = d1; p2 = d2; p3 = d3;
              } else {
                p0 = ex2_approx(d0); p1 = ex2_approx(d1);
                p2 = ex2_approx(d2); p3 = ex2_approx(d3);
              }
              acc2(sa, sb, p0, p1);
              acc2(sc, sd, p2, p3);
              pk[gi * 16 + c / 2] = pack_bf16x2(p0, p1);
              pk[gi * 16 + c / 2 + 1] = pack_bf16x2(p2, p3);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[gi * 16 + i] = 0u;
          }
        }
        l += (sa + sb) + (sc + sd);
        if (C::SEP_P && h == 0 && g_step > 0) {
          // P is about to be rewritten and O may be rescaled: the previous
          // P V of this slot must have finished.
          if (!warp_wait(&B.pv_done, (g_step - 1) & 1, &ctl->abort)) return;
          tc_fence_after();
        }
        __syncwarp();
        tmem_st32_wait(t_p + 32 * h, pk);
      }
      // O holds the P V of every earlier step (with P over S, this step's S
      // being ready means the previous P V has completed); bring it to the
      // new maximum before this step's P V adds to it.
      if (__any_sync(0xffffffffu, osc != 1.f)) {
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t w[32];
          __syncwarp();
          tmem_ld32_wait(t_o + c0, w);
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * osc);
          tmem_st32_wait(t_o + c0, w);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.p_full);
    }

    // Epilogue: O / l in bf16 and LSE = (m + log2 l) ln 2, once the last P V
    // is done (an empty tile has no P V and stores O = 0, LSE = -inf).
    const long long bh = tile / a.G;
    const long long qtok = (tile - bh * a.G) * C::TM + row;
    uint4* orow = reinterpret_cast<uint4*>(a.O + (bh * a.N + qtok) * D);
    if (ti.cnt > 0) {
      if (!warp_wait(&B.o_full, o_seen & 1, &ctl->abort)) return;
      ++o_seen;
      tc_fence_after();
    }
    if (ti.nch > 1) {
      chunk_epilogue<D>(a, ti, t_o, m_used, l, row, wq, row_ok, orow, a.LSE + bh * a.N + qtok);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.t_empty[buf]);
      continue;
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t w[32];
      if (ti.cnt > 0) {
        __syncwarp();
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
    if (lane == 0) mbar_arrive(&B.t_empty[buf]);
  }
}

template <int BS, int D, bool POS, bool CAUSAL>
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
      SlotBars& B = ctl->sb[s];
      for (int b = 0; b < kTiRing; ++b) {
        mbar_init(&B.t_full[b], 1);
        mbar_init(&B.t_empty[b], 4 + 2);  // the slot's softmax warps, its producer, the MMA issuer
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(&B.q_full[b], 1);
        mbar_init(&B.q_empty[b], 1);
        mbar_init(&B.k_full[b], 1);
        mbar_init(&B.k_empty[b], 1);
        mbar_init(&B.v_full[b], 1);
        mbar_init(&B.v_empty[b], 1);
      }
      mbar_init(&B.s_full, 1);
      mbar_init(&B.p_full, 4);
      mbar_init(&B.o_full, 1);
      mbar_init(&B.s_free, 4);
      mbar_init(&B.pv_done, 1);
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

  if (warp < 4 * kSlots) {
    softmax_role<BS, D, POS, CAUSAL>(warp >> 2, args, ctl, bitmaps, tmem);
    __syncwarp();
  } else if (warp == kProdWarp || warp == kProdWarp + 2) {
    produce_role<BS, D>((warp - kProdWarp) >> 1, &tmQ, &tmK, &tmV, args, smem, ctl, bitmaps);
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if ((threadIdx.x & 31) == 0) mma_role<BS, D>(args, smem, ctl, tmem);
    __syncwarp();
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
