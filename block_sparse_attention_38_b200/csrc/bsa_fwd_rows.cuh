// bsa_fwd_rows.cuh -- row-tile forward kernel (every block size).
//
// A tile is 128 query rows = R = 128 / block_size consecutive block rows of
// one (b, h).  The kernel walks the union of the tile's column lists in steps
// of 128 keys (128 / block_size blocks gathered into one shared-memory stage):
//
//   S = Q K_step^T            tcgen05.mma, M=128 queries, N=128 keys, K=d
//   P = 2^(S*scale*log2e - m) one thread per query row, fp32, written back to
//                             TMEM as bf16 over the first half of S
//   O += P V_step             tcgen05.mma with A = P read from TMEM, N=d
//
// A block row that does not hold a block of the step gets P = 0 there and its
// statistics skip it, so every row sums exactly over its own blocks ("Block
// Sparse Attention with Log-Linear Complexity", section 3.3); the exponentials
// of such blocks are not evaluated (membership is uniform over a warp).
//
// One persistent CTA per SM runs two independent tile slots so that the
// tensor core works on one slot while the other slot's softmax runs.  Roles:
//   warps 0-3   softmax / epilogue of slot 0    warps 4-7  same, slot 1
//   warp 8 + s  bitmap builder + TMA producer of slot s
//   warp 10 + s tcgen05.mma issuer of slot s (warp 10 also owns the TMEM)
// TMEM: slot s uses columns [256 s, 256 s + 128) for S (P aliases the first
// 64) and [256 s + 128, 256 s + 128 + d) for the O accumulator.
//
// Work split (`schedule`): tiles whose estimated cost (longest row plus one
// step) exceeds half of a CTA's share -- the global rows of the local+global
// pattern -- are dealt out one per CTA first; the remaining tiles are cut into
// contiguous ranges that fill each CTA's leftover share.  The CTA's two slots
// take tiles from its list in turn through a shared-memory counter.
#pragma once

#include "bsa_common.cuh"

namespace bsa {
namespace rows {

constexpr int kThreads = 384;
constexpr int kSlots = 2;

template <int BS, int D>
struct Cfg {
  static constexpr int TM = 128;                 // query rows per tile
  static constexpr int R = TM / BS;              // block rows per tile
  static constexpr int NK = 128;                 // keys per step
  static constexpr int BPS = NK / BS;            // blocks per step
  static constexpr int KATOMS = D / 64;          // 128-byte column atoms of a D-wide row
  static constexpr int Q_BYTES = TM * D * 2;
  static constexpr int CH_BYTES = NK * D * 2;    // one K or V stage
  static constexpr int NKS = D == 64 ? 2 : 1;    // K stages per slot
  static constexpr int NVS = D == 64 ? 2 : 1;    // V stages per slot
  static constexpr int SLOT_KV = (NKS + NVS) * CH_BYTES;
  static constexpr int OFF_Q = 0;                // + slot * Q_BYTES
  static constexpr int OFF_KV = kSlots * Q_BYTES;  // + slot * SLOT_KV: K stages, then V stages
  static constexpr int OFF_CTRL = OFF_KV + kSlots * SLOT_KV;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TMEM_SLOT = 256;
  static constexpr uint32_t TMEM_O = 128;
  static_assert((Q_BYTES % 1024) == 0 && (CH_BYTES % 1024) == 0, "1024-byte aligned stages");
};

struct SlotCtrl {
  uint64_t bm_full[2], bm_empty[2];
  uint64_t q_full, q_empty;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full, p_full, o_full, o_empty;
  uint64_t final_bar;
  long long tile[2];  // tile index of each bitmap buffer, -1 = no more work
  int n[2];           // union size (blocks) of each bitmap buffer
};

constexpr int kMaxGrid = 256;               // CTAs per launch (the host caps the grid)
constexpr int kMaxHeavyGroups = 2 * kMaxGrid;

// This CTA's work: up to two heavy tiles, then the light tiles of a
// contiguous range (heavy tiles inside it belong to other CTAs and are skipped).
struct Sched {
  long long heavy[2];
  long long light_begin, light_end;
  long long thr;                    // a tile group whose cost exceeds thr is heavy (-1: none is)
  long long scan[kThreads / 32];
  int n_heavy;
  int next_tile;                    // slots' shared cursor over heavy tiles, then light ones
  int light_next;
  int heavy_hg[kMaxHeavyGroups];    // heavy groups of one batch element, in order
  int heavy_cost[kMaxHeavyGroups];
};

struct Ctrl {
  SlotCtrl slot[kSlots];
  Sched sched;
  uint32_t tmem_base;
  AbortFlag abort;
  uint32_t bitmap[kSlots][2][5 * kMaxBitmapWords];  // R block-row maps, then their union
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
//  1. total = sum of all tile costs; a group is heavy when its cost exceeds
//     thr = total / (2*grid), half of one CTA's share (so there are fewer than
//     2*grid heavy tiles).
//  2. Heavy tile k (in tile order) goes to CTA k mod grid.
//  3. CTA c gets light capacity max(0, total/grid - its heavy cost); the light
//     tiles are cut into contiguous ranges whose light-cost prefix falls in
//     [L*Cap(c)/Cap, L*Cap(c+1)/Cap), Cap(c) the capacity of the CTAs before c.
// The busiest CTA then carries at most max(its heavy tiles, share + one light
// tile) instead of share + the largest tile.
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

  long long n_hv = 0, lsum = 0;
  for (long long hg = lo; hg < hi; ++hg) {
    const long long cst = group_cost<BS>(a, hg);
    if (cst > thr) ++n_hv; else lsum += cst;
  }
  long long Kg, Lper;
  long long hexcl = block_scan(n_hv, &Kg, sd.scan);
  const long long lexcl = block_scan(lsum, &Lper, sd.scan);
  for (long long hg = lo; hg < hi && n_hv > 0; ++hg) {
    const long long cst = group_cost<BS>(a, hg);
    if (cst > thr) {
      sd.heavy_hg[hexcl] = static_cast<int>(hg);
      sd.heavy_cost[hexcl] = static_cast<int>(cst);
      ++hexcl;
    }
  }
  __syncthreads();
  const long long Kh = Kg * nb;  // heavy tiles; Kh < 2*grid <= kMaxHeavyGroups
  auto heavy_tile_cost = [&](long long k) -> long long { return k < Kh ? sd.heavy_cost[k % Kg] : 0; };

  // Light capacity of the CTAs before this one, and of all of them.
  const long long target = total / grid;
  long long cap_before = 0, cap_all = 0, cap_mine = 0;
  for (long long cc = tid; cc < grid; cc += kThreads) {
    const long long hc = heavy_tile_cost(cc) + heavy_tile_cost(cc + grid);
    const long long cap = hc < target ? target - hc : 0;
    if (cc < c) cap_before += cap;
    if (cc == c) cap_mine = cap;
    cap_all += cap;
  }
  long long cap_b, cap_t, cap_m;
  block_scan(cap_before, &cap_b, sd.scan);
  block_scan(cap_all, &cap_t, sd.scan);
  block_scan(cap_mine, &cap_m, sd.scan);

  const long long L = Lper * nb;
  for (int e = 0; e < 2; ++e) {
    const long long capx = cap_b + (e ? cap_m : 0);
    long long x;
    if (c + e == grid) x = L;
    else if (cap_t > 0) x = static_cast<long long>(static_cast<__int128>(capx) * L / cap_t);
    else x = static_cast<long long>(static_cast<__int128>(c + e) * L / grid);
    long long* out = e == 0 ? &sd.light_begin : &sd.light_end;
    if (x >= L) {
      if (tid == 0) *out = a.num_tiles;
      continue;
    }
    const long long b = x / Lper, rem = x - b * Lper;
    if (rem == 0) {
      if (tid == 0) *out = b * HG;
      continue;
    }
    if (lexcl < rem && rem <= lexcl + lsum) {
      long long run = lexcl, hg = lo;
      while (run < rem) {
        const long long cst = group_cost<BS>(a, hg++);
        run += cst > thr ? 0 : cst;
      }
      *out = b * HG + hg;
    }
  }
  if (tid == 0) {
    int nh = 0;
    for (long long k = c; k < Kh && nh < 2; k += grid)
      sd.heavy[nh++] = (k / Kg) * HG + sd.heavy_hg[k % Kg];
    sd.n_heavy = nh;
    sd.thr = Kh > 0 ? thr : -1;  // -1: no heavy tile exists, nothing to skip
    sd.next_tile = 0;
    sd.light_next = 0;
  }
  __syncthreads();
}

// Next tile for a slot of this CTA (producer lane 0), -1 when none is left.
template <int BS>
__device__ __forceinline__ long long next_tile(const FwdArgs& a, Sched& sd) {
  const int i = atomicAdd(&sd.next_tile, 1);
  if (i < sd.n_heavy) return sd.heavy[i];
  const long long HG = static_cast<long long>(a.H) * a.G;
  for (;;) {
    const long long t = sd.light_begin + atomicAdd(&sd.light_next, 1);
    if (t >= sd.light_end) return -1;
    if (sd.thr < 0 || group_cost<BS>(a, t % HG) <= sd.thr) return t;
  }
}

// ------------------------------------------------------------ producer warp
template <int BS, int D>
__device__ void load_role(int s, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                          const CUtensorMap* tmV, const FwdArgs& a, uint8_t* smem, Ctrl* ctl) {
  using C = Cfg<BS, D>;
  SlotCtrl& sc = ctl->slot[s];
  const int lane = threadIdx.x & 31;
  uint8_t* q_s = smem + C::OFF_Q + s * C::Q_BYTES;
  uint8_t* k_s = smem + C::OFF_KV + s * C::SLOT_KV;
  uint8_t* v_s = k_s + C::NKS * C::CH_BYTES;
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
      w_ok = wait_bounded(&sc.bm_empty[buf], ((t >> 1) & 1) ^ 1, &ctl->abort);
      if (w_ok) {
        tile = next_tile<BS>(a, ctl->sched);
      }
    }
    if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
    tile = __shfl_sync(0xffffffffu, tile, 0);

    uint32_t* bm = ctl->bitmap[s][buf];
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
      sc.tile[buf] = tile;
      sc.n[buf] = n;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sc.bm_full[buf]);
    if (tile < 0) break;
    if (n == 0) continue;

    if (lane == 0) {
      const int g = static_cast<int>(tile - bh * a.G);
      ok = wait_bounded(&sc.q_empty, (q_loads & 1) ^ 1, &ctl->abort);
      if (ok) {
        mbar_arrive_expect_tx(&sc.q_full, C::Q_BYTES);
#pragma unroll
        for (int ka = 0; ka < C::KATOMS; ++ka)
          tma_load_3d(q_s + ka * (C::TM * 128), tmQ, &sc.q_full, ka * 64, g * C::TM,
                      static_cast<int>(bh));
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
        ok = wait_bounded(&sc.k_empty[ks], ((k_loads / C::NKS) & 1) ^ 1, &ctl->abort);
        if (!ok) break;
        mbar_arrive_expect_tx(&sc.k_full[ks], C::CH_BYTES);
#pragma unroll
        for (int b = 0; b < C::BPS; ++b)
#pragma unroll
          for (int ka = 0; ka < C::KATOMS; ++ka)
            tma_load_3d(k_s + ks * C::CH_BYTES + ka * (C::NK * 128) + b * (BS * 128), tmK,
                        &sc.k_full[ks], ka * 64, row0[b], static_cast<int>(bh));
        ++k_loads;
        const uint32_t vs = v_loads % C::NVS;
        ok = wait_bounded(&sc.v_empty[vs], ((v_loads / C::NVS) & 1) ^ 1, &ctl->abort);
        if (!ok) break;
        mbar_arrive_expect_tx(&sc.v_full[vs], C::CH_BYTES);
#pragma unroll
        for (int b = 0; b < C::BPS; ++b)
#pragma unroll
          for (int ka = 0; ka < C::KATOMS; ++ka)
            tma_load_3d(v_s + vs * C::CH_BYTES + ka * (C::NK * 128) + b * (BS * 128), tmV,
                        &sc.v_full[vs], ka * 64, row0[b], static_cast<int>(bh));
        ++v_loads;
      }
    }
    if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { ok = false; break; }
  }
  // On an early exit, let every copy already issued land before the CTA ends.
  if (!ok && lane == 0) {
    if (q_loads > 0) wait_drain(&sc.q_full, (q_loads - 1) & 1);
    for (uint32_t st = 0; st < C::NKS; ++st)
      if (k_loads > st) {
        const uint32_t last = st + C::NKS * ((k_loads - 1 - st) / C::NKS);
        wait_drain(&sc.k_full[st], (last / C::NKS) & 1);
      }
    for (uint32_t st = 0; st < C::NVS; ++st)
      if (v_loads > st) {
        const uint32_t last = st + C::NVS * ((v_loads - 1 - st) / C::NVS);
        wait_drain(&sc.v_full[st], (last / C::NVS) & 1);
      }
  }
  __syncwarp();
}

// ---------------------------------------------------------------- MMA issuer
// Per step: S = Q K^T, then (once the softmax has written P) O += P V.  The
// QK of the next step is issued right after the PV of this one: MMAs of one
// thread run in issue order, so it overwrites S/P only after the PV read P,
// and the commit that reports it also reports that PV.
template <int BS, int D>
__device__ void mma_role(int s, const FwdArgs& a, uint8_t* smem, Ctrl* ctl, uint32_t tmem) {
  using C = Cfg<BS, D>;
  SlotCtrl& sc = ctl->slot[s];
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, C::NK, false, false);  // Q, K K-major
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);       // V MN-major
  const uint32_t q_base = smem_u32(smem + C::OFF_Q + s * C::Q_BYTES);
  const uint32_t k_base = smem_u32(smem + C::OFF_KV + s * C::SLOT_KV);
  const uint32_t v_base = k_base + C::NKS * C::CH_BYTES;
  const uint32_t t_s = tmem + s * C::TMEM_SLOT;
  const uint32_t t_o = t_s + C::TMEM_O;
  uint32_t k_cons = 0, v_cons = 0, q_uses = 0, p_seen = 0, o_tiles = 0;
  bool ok = true;
  for (int t = 0; ok; ++t) {
    const int buf = t & 1;
    if (!wait_bounded(&sc.bm_full[buf], (t >> 1) & 1, &ctl->abort)) break;
    const long long tile = sc.tile[buf];
    const int n = sc.n[buf];
    mbar_arrive(&sc.bm_empty[buf]);
    if (tile < 0) break;
    if (n == 0) continue;
    const int steps = (n + C::BPS - 1) / C::BPS;
    if (!wait_bounded(&sc.q_full, q_uses & 1, &ctl->abort)) break;
    ++q_uses;
    for (int j = 0; j < steps; ++j) {
      const uint32_t ks = k_cons % C::NKS;
      if (!wait_bounded(&sc.k_full[ks], (k_cons / C::NKS) & 1, &ctl->abort)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t ad = sdesc_sw128(q_base + (kk >> 2) * (C::TM * 128) + (kk & 3) * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(
            k_base + ks * C::CH_BYTES + (kk >> 2) * (C::NK * 128) + (kk & 3) * 32, 16, 1024);
        umma_bf16_ss(t_s, ad, bd, kIdescQK, kk > 0 ? 1u : 0u);
      }
      umma_commit(&sc.k_empty[ks]);
      umma_commit(&sc.s_full);
      if (j == steps - 1) umma_commit(&sc.q_empty);
      ++k_cons;

      if (!wait_bounded(&sc.p_full, p_seen & 1, &ctl->abort)) { ok = false; break; }
      ++p_seen;
      const uint32_t vs = v_cons % C::NVS;
      if (!wait_bounded(&sc.v_full[vs], (v_cons / C::NVS) & 1, &ctl->abort)) { ok = false; break; }
      if (j == 0 && o_tiles > 0 &&
          !wait_bounded(&sc.o_empty, (o_tiles - 1) & 1, &ctl->abort)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < C::NK / 16; ++kk) {
        const uint64_t bd =
            sdesc_sw128(v_base + vs * C::CH_BYTES + kk * (16 * 128), C::NK * 128, 1024);
        umma_bf16_ts(t_o, t_s + kk * 8, bd, kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&sc.v_empty[vs]);
      ++v_cons;
      if (j == steps - 1) umma_commit(&sc.o_full);
    }
    ++o_tiles;
  }
  // Every MMA issued must complete before the TMEM is released.
  umma_commit(&sc.final_bar);
  wait_drain(&sc.final_bar, 0);
}

// ------------------------------------------------------------ softmax warps
template <int BS, int D>
__device__ void softmax_role(int s, const FwdArgs& a, Ctrl* ctl, uint32_t tmem) {
  using C = Cfg<BS, D>;
  SlotCtrl& sc = ctl->slot[s];
  const int row = threadIdx.x - s * 128;  // query row of the tile
  const int warp = row >> 5;
  const int lane = row & 31;
  const int sub = row / BS;               // block row of the tile this thread belongs to
  const int qq = row % BS;                // position inside that block row
  const uint32_t t_s = tmem + s * C::TMEM_SLOT + (static_cast<uint32_t>(warp * 32) << 16);
  const uint32_t t_o = t_s + C::TMEM_O;
  const float sl2 = a.scale_log2;
  constexpr float kNegInf = -INFINITY;
  uint32_t s_seen = 0, o_seen = 0;

  for (int t = 0;; ++t) {
    const int buf = t & 1;
    if (!warp_wait(&sc.bm_full[buf], (t >> 1) & 1, &ctl->abort)) return;
    const long long tile = sc.tile[buf];
    const int n = sc.n[buf];
    if (tile < 0) return;
    const uint32_t* bm = ctl->bitmap[s][buf];
    const uint32_t* mine = bm + sub * a.W;
    const long long bh = tile / a.G;
    const int g = static_cast<int>(tile - bh * a.G);
    const int r_sub = g * C::R + sub;
    const bool row_ok = r_sub < a.M;
    const int steps = (n + C::BPS - 1) / C::BPS;

    float m_used = kNegInf;  // running max, log2 units of the scaled score
    float l = 0.f;           // running sum of 2^(s - m_used)
    BitIter it(bm + C::R * a.W, a.W);
    for (int j = 0; j < steps; ++j) {
      // Blocks of this step: vmask bit b = this row holds block b of the step,
      // dmask bit b = block b is this row's diagonal block under causal masking.
      uint32_t vmask = 0, dmask = 0;
#pragma unroll
      for (int b = 0; b < C::BPS; ++b) {
        const int jb = it.next();
        if (row_ok && jb >= 0 && ((mine[jb >> 5] >> (jb & 31)) & 1u)) vmask |= 1u << b;
        if (a.causal && jb == r_sub) dmask |= 1u << b;
      }
      if (!warp_wait(&sc.s_full, s_seen & 1, &ctl->abort)) return;
      ++s_seen;
      tc_fence_after();
      // The 128 scores are taken in four groups of 32 columns (group g covers
      // keys 32g..32g+31, block g*32/BS); a group is read from TMEM once for
      // the maximum and once for the exponentials, and its 16 packed P
      // columns are written over S columns already consumed.
      if (vmask != 0) {  // uniform over the warp
        float mx = kNegInf;
#pragma unroll 1
        for (int gp = 0; gp < 2; ++gp) {
          const int b0 = (2 * gp) * 32 / BS, b1 = (2 * gp + 1) * 32 / BS;
          const bool ok0 = (vmask >> b0) & 1u, ok1 = (vmask >> b1) & 1u;
          if (!ok0 && !ok1) continue;
          uint32_t u[64];
          tmem_ld32(t_s + gp * 64, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          tmem_ld32(t_s + gp * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          tmem_wait_ld();
          reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&u[32]));
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int b = h ? b1 : b0;
            if (!(h ? ok1 : ok0)) continue;
            const bool diag = (dmask >> b) & 1u;
            const int c0 = ((2 * gp + h) * 32) % BS;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              float v = __uint_as_float(u[h * 32 + i]) * sl2;
              if (diag && c0 + i > qq) v = kNegInf;
              mx = fmaxf(mx, v);
            }
          }
        }
        float factor = 1.f;
        bool need_rescale = false;
        const float m_new = fmaxf(m_used, mx);
        if (m_new > m_used + kRescaleThreshold) {
          if (l > 0.f) {
            need_rescale = true;
            factor = ex2_approx(m_used - m_new);
          }
          m_used = m_new;
        }
        // The commit behind s_full also covers the previous PV: O is final here.
        if (__any_sync(0xffffffffu, need_rescale)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t u[32];
            tmem_ld32(t_o + c * 32, u);
            tmem_wait_ld();
            reg_fence32(u);
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * factor);
            tmem_st32(t_o + c * 32, u);
          }
        }
        const float mu = m_used == kNegInf ? 0.f : m_used;
        float rs = 0.f;
#pragma unroll 1
        for (int gp = 0; gp < 2; ++gp) {
          const int b0 = (2 * gp) * 32 / BS, b1 = (2 * gp + 1) * 32 / BS;
          const bool ok0 = (vmask >> b0) & 1u, ok1 = (vmask >> b1) & 1u;
          uint32_t pk[32];
          uint32_t u[64];
          if (ok0 || ok1) {
            tmem_ld32(t_s + gp * 64, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
            tmem_ld32(t_s + gp * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
            tmem_wait_ld();
            reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&u[0]));
            reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int b = h ? b1 : b0;
            if (h ? ok1 : ok0) {
              const bool diag = (dmask >> b) & 1u;
              const int c0 = ((2 * gp + h) * 32) % BS;
#pragma unroll
              for (int i = 0; i < 32; i += 2) {
                float v0 = __uint_as_float(u[h * 32 + i]) * sl2, v1 = __uint_as_float(u[h * 32 + i + 1]) * sl2;
                if (diag && c0 + i > qq) v0 = kNegInf;
                if (diag && c0 + i + 1 > qq) v1 = kNegInf;
                const float p0 = ex2_approx(v0 - mu), p1 = ex2_approx(v1 - mu);
                rs += p0;
                rs += p1;
                pk[h * 16 + i / 2] = pack_bf16x2(p0, p1);
              }
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[h * 16 + i] = 0u;
            }
          }
          tmem_st32(t_s + gp * 32, pk);
        }
        l = l * factor + rs;
      } else {
        uint32_t z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0u;
        tmem_st32(t_s, z);
        tmem_st32(t_s + 32, z);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sc.p_full);
    }

    // Epilogue: O / l in bf16 and LSE = (m + log2 l) ln 2.
    const long long qtok = static_cast<long long>(g) * C::TM + row;
    __nv_bfloat16* orow = a.O + (bh * a.N + qtok) * D;
    if (n > 0) {
      if (!warp_wait(&sc.o_full, o_seen & 1, &ctl->abort)) return;
      ++o_seen;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(t_o + c * 32, u);
        tmem_wait_ld();
        reg_fence32(u);
        if (row_ok) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(u[q * 8 + 0]) * inv, __uint_as_float(u[q * 8 + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(u[q * 8 + 2]) * inv, __uint_as_float(u[q * 8 + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(u[q * 8 + 4]) * inv, __uint_as_float(u[q * 8 + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(u[q * 8 + 6]) * inv, __uint_as_float(u[q * 8 + 7]) * inv);
            dst[c * 4 + q] = v;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sc.o_empty);
      if (row_ok)
        a.LSE[bh * a.N + qtok] = l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994531f : kNegInf;
    } else if (row_ok) {
      uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
      a.LSE[bh * a.N + qtok] = kNegInf;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sc.bm_empty[buf]);
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
    for (int s = 0; s < kSlots; ++s) {
      SlotCtrl& sc = ctl->slot[s];
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sc.bm_full[b], 1);
        mbar_init(&sc.bm_empty[b], 5);  // four softmax warps + the MMA issuer
        mbar_init(&sc.k_full[b], 1);
        mbar_init(&sc.k_empty[b], 1);
        mbar_init(&sc.v_full[b], 1);
        mbar_init(&sc.v_empty[b], 1);
      }
      mbar_init(&sc.q_full, 1);
      mbar_init(&sc.q_empty, 1);
      mbar_init(&sc.s_full, 1);
      mbar_init(&sc.p_full, 4);
      mbar_init(&sc.o_full, 1);
      mbar_init(&sc.o_empty, 4);
      mbar_init(&sc.final_bar, 1);
    }
    ctl->abort.v = 0;
    fence_mbar_init();
  }
  if (warp == 10) {
    tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  schedule<BS>(args, ctl);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp < 8) {
    softmax_role<BS, D>(warp >> 2, args, ctl, tmem);
    __syncwarp();
  } else {
    if (warp < 10) {
      load_role<BS, D>(warp - 8, &tmQ, &tmK, &tmV, args, smem, ctl);
    } else {
      if ((threadIdx.x & 31) == 0) mma_role<BS, D>(warp - 10, args, smem, ctl, tmem);
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 10) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace rows
}  // namespace bsa
